// tconv.cu -- the Mix-FFN temporal convolution with its last-frame cache
// (lin_attn_temporal_conv in include/linattn.h).
//
// SANA-Video paper-graph page, "Spatial-Temporal Mix-FFN" and "Block Causal
// Mix-FFN": a kernel-3 convolution along the frame axis of the block's hidden
// states, added back through a shortcut, with the zero frame after the block
// and the previous block's cached last frame before it.
//
// The op moves each element once in and once out (about 0.4 flop per byte),
// so it is bound by HBM bandwidth: one thread owns a 16-byte vector of
// channels at one spatial position and walks the frames, keeping frames t-1,
// t, t+1 in registers and loading kAhead frames ahead so that every thread
// has several independent 16-byte loads in flight. Consecutive threads take
// consecutive channel vectors, so each frame's loads and stores are
// contiguous across a warp. The grid strides over the columns, sized to fill
// every SM.
#include "linattn.h"

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kThreads = 128;
constexpr int kAhead = 4;           // frames whose loads a thread issues together
constexpr int kBlocksPerSm = 16;

template <typename T>
struct Lanes;
template <>
struct Lanes<float> {
  static constexpr int V = 4;       // channels per 16-byte vector
};
template <>
struct Lanes<__nv_bfloat16> {
  static constexpr int V = 8;
};

__device__ __forceinline__ void unpack(const uint4& r, float (&f)[4]) {
  f[0] = __uint_as_float(r.x);
  f[1] = __uint_as_float(r.y);
  f[2] = __uint_as_float(r.z);
  f[3] = __uint_as_float(r.w);
}

__device__ __forceinline__ void unpack(const uint4& r, float (&f)[8]) {
  const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);            // low half: even channel
    f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 pack(const float (&f)[4]) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);   // round to nearest even
  return reinterpret_cast<const uint32_t&>(h);
}

__device__ __forceinline__ uint4 pack(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

template <int V>
__device__ __forceinline__ void load_taps(const float* __restrict__ p, float (&f)[V]) {
#pragma unroll
  for (int i = 0; i < V; i += 4) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p + i));
    f[i] = a.x;
    f[i + 1] = a.y;
    f[i + 2] = a.z;
    f[i + 3] = a.w;
  }
}

// One column = (b, s, channel vector); cols = B * S * C / V.
template <typename T>
__global__ void __launch_bounds__(kThreads)
temporal_conv_kernel(const T* __restrict__ x, const float* __restrict__ w,
                     const float* __restrict__ bias, const T* cache_in, T* __restrict__ y,
                     T* cache_out, int nT, long long S, int C, long long cols) {
  constexpr int V = Lanes<T>::V;
  const int CV = C / V;
  const long long frame = S * (long long)C;    // elements per frame
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long col = (long long)blockIdx.x * blockDim.x + threadIdx.x; col < cols;
       col += stride) {
    const int cv = (int)(col % CV);
    const long long bs = col / CV;               // b * S + s
    const long long b = bs / S;
    const long long s = bs - b * S;
    const int c0 = cv * V;

    float w0[V], w1[V], w2[V], bb[V];
    load_taps<V>(w + c0, w0);
    load_taps<V>(w + C + c0, w1);
    load_taps<V>(w + 2 * C + c0, w2);
    if (bias) {
      load_taps<V>(bias + c0, bb);
    } else {
#pragma unroll
      for (int i = 0; i < V; ++i) bb[i] = 0.f;
    }

    const long long base = (b * nT * S + s) * C + c0;     // frame 0 of the column
    const long long cbase = bs * C + c0;                   // the column in a cache frame
    float prev[V], cur[V], nxt[V];
    if (cache_in) {
      unpack(*reinterpret_cast<const uint4*>(cache_in + cbase), prev);
    } else {
#pragma unroll
      for (int i = 0; i < V; ++i) prev[i] = 0.f;
    }
    uint4 last = __ldg(reinterpret_cast<const uint4*>(x + base));
    unpack(last, cur);
    for (int t0 = 0; t0 < nT; t0 += kAhead) {
      uint4 raw[kAhead];
#pragma unroll
      for (int i = 0; i < kAhead; ++i) {
        const int t = t0 + 1 + i;
        raw[i] = t < nT ? __ldg(reinterpret_cast<const uint4*>(x + base + t * frame))
                        : make_uint4(0u, 0u, 0u, 0u);     // the zero frame after the block
      }
#pragma unroll
      for (int i = 0; i < kAhead; ++i) {
        const int t = t0 + i;
        if (t < nT) {
          unpack(raw[i], nxt);
          float o[V];
#pragma unroll
          for (int j = 0; j < V; ++j) {
            float a = cur[j] + bb[j];
            a = fmaf(w0[j], prev[j], a);
            a = fmaf(w1[j], cur[j], a);
            a = fmaf(w2[j], nxt[j], a);
            o[j] = a;
          }
          *reinterpret_cast<uint4*>(y + base + t * frame) = pack(o);
          if (t + 1 < nT) last = raw[i];
#pragma unroll
          for (int j = 0; j < V; ++j) {
            prev[j] = cur[j];
            cur[j] = nxt[j];
          }
        }
      }
    }
    // the block's last input frame, bit for bit, becomes the next block's cache
    if (cache_out) *reinterpret_cast<uint4*>(cache_out + cbase) = last;
  }
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
  return a0 < b0 + nb && b0 < a0 + na;
}

}  // namespace

extern "C" la_status lin_attn_temporal_conv(int B, int T, int S, int C, la_dtype dtype,
                                            const void* x, const float* weight,
                                            const float* bias, const void* cache_in, void* y,
                                            void* cache_out, void* stream) {
  if (B < 0 || T < 0 || S < 0 || C < 0) return LA_ERR_INVALID_ARG;
  if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
  const size_t elt = dtype == LA_BF16 ? 2 : 4;
  const int V = (int)(16 / elt);
  if (C % V != 0) return LA_ERR_INVALID_ARG;
  const long long n = (long long)B * T * S * C;
  if (n == 0) return LA_OK;
  if (!x || !y || !weight) return LA_ERR_INVALID_ARG;
  const void* ptrs[6] = {x, weight, bias, cache_in, y, cache_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return LA_ERR_INVALID_ARG;
  const size_t xb = (size_t)n * elt;
  const size_t cb = (size_t)B * S * C * elt;
  const size_t wb = (size_t)3 * C * sizeof(float), bb = (size_t)C * sizeof(float);
  if (overlaps(y, xb, x, xb) || overlaps(y, xb, weight, wb) || overlaps(y, xb, bias, bb) ||
      overlaps(y, xb, cache_in, cb) || overlaps(y, xb, cache_out, cb))
    return LA_ERR_INVALID_ARG;
  if (overlaps(cache_out, cb, x, xb) || overlaps(cache_out, cb, weight, wb) ||
      overlaps(cache_out, cb, bias, bb) ||
      (cache_out != cache_in && overlaps(cache_out, cb, cache_in, cb)))
    return LA_ERR_INVALID_ARG;

  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  const long long cols = (long long)B * S * C / V;     // (b, s, channel vector) columns
  long long blocks = (cols + kThreads - 1) / kThreads;
  const long long cap = (long long)sms * kBlocksPerSm;
  if (blocks > cap) blocks = cap;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == LA_BF16) {
    temporal_conv_kernel<__nv_bfloat16><<<(unsigned)blocks, kThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), weight, bias,
        static_cast<const __nv_bfloat16*>(cache_in), static_cast<__nv_bfloat16*>(y),
        static_cast<__nv_bfloat16*>(cache_out), T, S, C, cols);
  } else {
    temporal_conv_kernel<float><<<(unsigned)blocks, kThreads, 0, st>>>(
        static_cast<const float*>(x), weight, bias, static_cast<const float*>(cache_in),
        static_cast<float*>(y), static_cast<float*>(cache_out), T, S, C, cols);
  }
  if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
  return LA_OK;
}

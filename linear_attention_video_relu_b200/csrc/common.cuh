// common.cuh -- types and device helpers shared by the kernels of liblinattn.
//
// The operation is ReLU linear attention with RoPE applied after the ReLU in
// the numerator only (SANA-Video paper-graph page, section 3.4, Eq. 2), with
// the state (S, z) of "Block Linear Attention with Constant-Memory KV Cache"
// (Eq. 3, Algorithm 1) carried across blocks of frames.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace la {

// Upper bound on the cos/sin table of one call (float2 entries, 48 KB).
constexpr int kMaxRopeEntries = 6144;

// Division by a runtime constant d >= 1 for dividends 0 <= n < 2^31:
// n / d == (n * m) >> p with p = 31 + ceil(log2 d), m = ceil(2^p / d) (the
// rounding-up method of Granlund and Montgomery, exact in this range).
struct FastDiv {
  unsigned long long m;
  int p;
  int d;
};

inline FastDiv make_fastdiv(int d) {
  FastDiv f;
  int l = 0;
  while ((1LL << l) < d) ++l;
  f.p = 31 + l;
  f.m = (unsigned long long)((((unsigned __int128)1 << f.p) + (unsigned)d - 1) / (unsigned)d);
  f.d = d;
  return f;
}

__host__ __device__ __forceinline__ int fdiv(const FastDiv& f, int n) {
  return (int)(((unsigned long long)(unsigned)n * f.m) >> f.p);
}

// Geometry of the 3D rotary embedding for one call. The D dims are split into
// t | h | w segments; segment a holds half[a] rotation pairs. The table holds
// (cos, sin) for every (axis, position, pair): t positions are the call's
// frames t_offset .. t_offset + T - 1, h and w positions 0 .. Hg-1 / Wg-1.
struct Rope {
  int on;
  int T, Hg, Wg;
  int t_offset;
  int half[3];       // pairs per axis (d_axis / 2)
  int stride[3];     // table row length per position (rope_stride(half))
  int pair_base[3];  // first pair index of each axis
  int tab_off[3];    // first table entry of each axis
  int entries;       // table size in float2
  double theta;
  FastDiv div_hw;    // by Hg * Wg
  FastDiv div_w;     // by Wg
  // theta^(-2m/d) / pi of every pair (pair order) as an unevaluated float sum
  // hi + lo, so that position * frequency / pi is formed to ~2^-48 relative
  float inv_pi_hi[64];
  float inv_pi_lo[64];
};

// Memory order of q, k, v, gate and out: [B, H, N, D] (bnhd = 0) or
// [B, N, H, D] (bnhd = 1, the order a fused QKV projection writes its heads
// in), D innermost either way; head = b * H + h.
struct Layout {
  int bnhd;
  int H;
  FastDiv div_h;   // by H
  // element offset of (head, token n, dim 0) in a tensor of N tokens per head
  // and rows of D values
  __host__ __device__ __forceinline__ long long row(int head, long long n, long long N,
                                                    int D) const {
    if (!bnhd) return ((long long)head * N + n) * D;
    const int b = fdiv(div_h, head), h = head - b * H;
    return (((long long)b * N + n) * H + h) * D;
  }
  // elements between consecutive tokens of one head
  __host__ __device__ __forceinline__ long long tok_stride(int D) const {
    return bnhd ? (long long)H * D : (long long)D;
  }
};

// Work schedule of the state build. The tokens of every head are cut into
// segments of L tokens (the whole head in bidirectional mode, one block in
// block-causal mode); a segment is cut into tps tiles of TT tokens (the last
// one ragged). The U = nseg * tps tiles, in order, are dealt out to G CTAs as
// contiguous ranges [floor(i U / G), floor((i+1) U / G)). A CTA writes one
// partial state per segment it touches, into slot
// seg * maxc + (i - first CTA of seg), so the reduction can sum the partials
// of a segment in CTA order without atomics.
struct Sched {
  long long U;
  int G;
  int tps;
  int TT;
  int L;
  int nblk;   // segments per head
  int nseg;
  int maxc;
  int fastU;       // U * G < 2^31: divU divides tile products exactly
  FastDiv divU;
};

__host__ __device__ inline long long unit_begin(const Sched& s, long long i) {
  return i * s.U / s.G;
}

// The CTA whose range holds tile u: the largest i with unit_begin(i) <= u.
__host__ __device__ inline int cta_of_unit(const Sched& s, long long u) {
  return (int)(((u + 1) * (long long)s.G - 1) / s.U);
}

// cta_of_unit with one multiply-shift when U * G < 2^31.
__host__ __device__ __forceinline__ int cta_of_unit_fast(const Sched& s, long long u) {
  return s.fastU ? fdiv(s.divU, (int)((u + 1) * s.G - 1)) : cta_of_unit(s, u);
}

// Number of CTAs (= partial slots) that hold tiles of segment seg.
__host__ __device__ __forceinline__ int parts_of(const Sched& s, int seg) {
  const long long ub = (long long)seg * s.tps;
  return cta_of_unit_fast(s, ub + s.tps - 1) - cta_of_unit_fast(s, ub) + 1;
}

__host__ __device__ inline long long slot_index(const Sched& s, int seg, int cta) {
  return (long long)seg * s.maxc + (cta - cta_of_unit(s, (long long)seg * s.tps));
}

// ---- RoPE table ----------------------------------------------------------
//
// One row per (axis, position); a row of an axis with `half` rotation pairs
// holds G = ceil(half / 4) groups of 8 floats -- cos of pairs 4g .. 4g+3, then
// their sin -- and 4 padding floats, so that a row spans an odd number of
// 16-byte units (conflict-free 16-byte loads of consecutive positions). Pairs
// past `half` in the last group read cos 1, sin 0. Sizes and offsets (stride,
// tab_off, entries) count float2 units of 8 bytes.

// Row length in float2 units for an axis with `half` pairs (0 for none).
__host__ __device__ inline int rope_stride(int half) {
  return half == 0 ? 0 : 4 * ((half + 3) / 4) + 2;
}

// cos, sin of pair m at position pos on axis a: the angle pos * theta^(-2m/d)
// with x = angle / pi carried as x_hi + x_lo (the product error of x_hi
// recovered exactly by an FMA); x_hi - 2 rint(x_hi / 2) is exact, so the
// reduced argument in [-1, 1] is accurate to a few ulp and sincospif gives
// cos, sin to float precision. ih / il: theta^(-2m/d) / pi of every pair as a
// float sum hi + lo, in shared memory (a parameter-space read of a per-lane
// index would be serialised).
__device__ inline void rope_angle_cs(int pos, int pair, const float* ih, const float* il,
                                     float& c, float& s) {
  const float P = (float)pos;                         // exact: positions < 2^24
  const float x_hi = P * ih[pair];
  const float x_lo = fmaf(P, ih[pair], -x_hi) + P * il[pair];
  const float red = (x_hi - 2.f * rintf(0.5f * x_hi)) + x_lo;
  sincospif(red, &s, &c);
}

// Fills the whole table (threads tid, tid + nthr, ...): one work item per
// (axis, position, group), the item g == G writing the row's padding.
__device__ inline void rope_fill(const Rope& r, const float* ih, const float* il, float* tab,
                                 int tid, int nthr) {
  const int G0 = (r.half[0] + 3) / 4, G1 = (r.half[1] + 3) / 4, G2 = (r.half[2] + 3) / 4;
  const int n0 = r.half[0] ? r.T * (G0 + 1) : 0;
  const int n1 = r.half[1] ? r.Hg * (G1 + 1) : 0;
  const int n2 = r.half[2] ? r.Wg * (G2 + 1) : 0;
  for (int it = tid; it < n0 + n1 + n2; it += nthr) {
    const int a = it < n0 ? 0 : (it < n0 + n1 ? 1 : 2);
    const int local = it - (a == 0 ? 0 : (a == 1 ? n0 : n0 + n1));
    const int Ga = a == 0 ? G0 : (a == 1 ? G1 : G2);
    const int half = a == 0 ? r.half[0] : (a == 1 ? r.half[1] : r.half[2]);
    const int pos = local / (Ga + 1);
    const int g = local - pos * (Ga + 1);
    const int toff = a == 0 ? r.tab_off[0] : (a == 1 ? r.tab_off[1] : r.tab_off[2]);
    const int stride = a == 0 ? r.stride[0] : (a == 1 ? r.stride[1] : r.stride[2]);
    const int pbase = a == 0 ? r.pair_base[0] : (a == 1 ? r.pair_base[1] : r.pair_base[2]);
    float* row = tab + 2 * (toff + pos * stride);
    if (g == Ga) {
      *reinterpret_cast<float4*>(row + 8 * g) = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    float cv[4], sv[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int m = 4 * g + w;
      cv[w] = 1.f;
      sv[w] = 0.f;
      if (m < half) rope_angle_cs(pos + (a == 0 ? r.t_offset : 0), pbase + m, ih, il, cv[w], sv[w]);
    }
    *reinterpret_cast<float4*>(row + 8 * g) = make_float4(cv[0], cv[1], cv[2], cv[3]);
    *reinterpret_cast<float4*>(row + 8 * g + 4) = make_float4(sv[0], sv[1], sv[2], sv[3]);
  }
}

// (cos, sin) of pair p (0 .. D/2-1) for a token at local frame tl, row h,
// column w.
__device__ inline float2 rope_cs(const Rope& r, const float* tab, int p, int tl, int h, int w) {
  const int ax = p < r.pair_base[1] ? 0 : (p < r.pair_base[2] ? 1 : 2);
  const int m = p - r.pair_base[ax];
  const int pos = ax == 0 ? tl : (ax == 1 ? h : w);
  const int i = 2 * (r.tab_off[ax] + pos * r.stride[ax]) + 8 * (m >> 2) + (m & 3);
  return make_float2(tab[i], tab[i + 4]);
}

// ---- element access --------------------------------------------------------

__device__ inline float to_f32(float x) { return x; }
__device__ inline float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ inline T from_f32(float x);
template <> __device__ inline float from_f32<float>(float x) { return x; }
template <> __device__ inline __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ inline float relu(float x) { return x > 0.f ? x : 0.f; }

__device__ inline float sigmoid(float x) { return 1.f / (1.f + expf(-x)); }

}  // namespace la

// simt.cuh -- CUDA-core kernels: the fp32 I/O path, the token-causal mode
// and every shape the tensor-core path does not take (D = 32, rope widths
// not multiples of 8).
//
// Three launches per call, each a step of the factorised form of Eq. 2
// (SANA-Video paper-graph page, section 3.4):
//   state_partial_simt  per tile range: S_part = sum RoPE(phi k)^T v, z_part = sum phi k
//   reduce_states       fixed-order sum of the partials (+ carried state, + block scan)
//   apply_simt          out = RoPE(phi q) S / (phi q . z + eps), times sigmoid(g)
//   (apply_causal_simt in token-causal mode)
#pragma once

#include "common.cuh"

namespace la {

constexpr int kSimtThreads = 256;
constexpr int kSimtTileState = 32;   // tokens per tile of the state build
constexpr int kSimtTileApply = 32;   // tokens per tile of the apply step
// Token-causal mode: segments (chunks) of this many tokens, one tile each.
constexpr int kCausalChunk = 32;
static_assert(kCausalChunk == kSimtTileState && kCausalChunk == kSimtTileApply,
              "a causal chunk is one tile of each kernel");

// Position (local frame, row, column) of token n of a head.
__device__ inline void token_pos(const Rope& r, long long n, int& tl, int& h, int& w) {
  long long hw = (long long)r.Hg * r.Wg;
  tl = (int)(n / hw);
  long long rem = n - (long long)tl * hw;
  h = (int)(rem / r.Wg);
  w = (int)(rem - (long long)h * r.Wg);
}

// Each CTA walks its contiguous range of tiles; a thread owns an (D/16) x
// (D/16) block of the D x D partial state in registers and threads 0..D-1 own
// one entry of z. Every CTA also writes its share of the RoPE table to
// `gtab` for the apply kernel.
template <int D, typename T>
__global__ void __launch_bounds__(kSimtThreads)
state_partial_simt(const T* __restrict__ k, const T* __restrict__ v, long long N,
                   Layout lay, Rope rope, Sched sc, float* __restrict__ partials,
                   float2* __restrict__ gtab) {
  constexpr int TT = kSimtTileState;
  constexpr int R = D / 16;
  constexpr int DD1 = D * (D + 1);
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* s_kr = reinterpret_cast<float*>(smem_raw);  // [TT][D] rotated phi(k)
  float* s_kphi = s_kr + TT * D;                     // [TT][D] phi(k)
  float* s_v = s_kphi + TT * D;                      // [TT][D]
  float2* s_tab = reinterpret_cast<float2*>(s_v + TT * D);
  const int tid = threadIdx.x;
  const int cta = blockIdx.x;

  if (rope.on) {
    __shared__ float s_ih[64], s_il[64];
    if (tid < D / 2) {
      s_ih[tid] = rope.inv_pi_hi[tid];
      s_il[tid] = rope.inv_pi_lo[tid];
    }
    __syncthreads();
    rope_fill(rope, s_ih, s_il, reinterpret_cast<float*>(s_tab), tid, kSimtThreads);
    __syncthreads();
    int e0 = (int)((long long)cta * rope.entries / gridDim.x);
    int e1 = (int)((long long)(cta + 1) * rope.entries / gridDim.x);
    for (int e = e0 + tid; e < e1; e += kSimtThreads) gtab[e] = s_tab[e];
  }

  const int ta = tid / 16, tc = tid % 16;
  float acc[R][R];
  float zacc = 0.f;
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int j = 0; j < R; ++j) acc[i][j] = 0.f;

  auto flush = [&](int seg) {
    float* slot = partials + slot_index(sc, seg, cta) * DD1;
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int j = 0; j < R; ++j) {
        slot[(ta * R + i) * D + tc * R + j] = acc[i][j];
        acc[i][j] = 0.f;
      }
    if (tid < D) slot[D * D + tid] = zacc;
    zacc = 0.f;
  };

  const long long u0 = unit_begin(sc, cta), u1 = unit_begin(sc, cta + 1);
  int cur = -1;
  for (long long u = u0; u < u1; ++u) {
    const int seg = (int)(u / sc.tps);
    const int tile = (int)(u - (long long)seg * sc.tps);
    if (seg != cur) {
      if (cur >= 0) flush(cur);
      cur = seg;
    }
    const int head = seg / sc.nblk, blk = seg - head * sc.nblk;
    const int r0 = tile * TT;
    // segments hold L tokens, except a ragged last chunk in token-causal mode
    const int seglen = (int)min((long long)sc.L, N - (long long)blk * sc.L);
    const int rows = min(TT, seglen - r0);
    const long long nbase = (long long)blk * sc.L + r0;
    const T* kh = k + lay.row(head, nbase, N, D);
    const T* vh = v + lay.row(head, nbase, N, D);
    const long long ts = lay.tok_stride(D);
    for (int idx = tid; idx < TT * (D / 2); idx += kSimtThreads) {
      const int r = idx / (D / 2), pr = idx - r * (D / 2);
      float x0 = 0.f, x1 = 0.f, v0 = 0.f, v1 = 0.f;
      if (r < rows) {
        x0 = relu(to_f32(kh[r * ts + 2 * pr]));
        x1 = relu(to_f32(kh[r * ts + 2 * pr + 1]));
        v0 = to_f32(vh[r * ts + 2 * pr]);
        v1 = to_f32(vh[r * ts + 2 * pr + 1]);
      }
      float y0 = x0, y1 = x1;
      if (rope.on && r < rows) {
        int tl, h, w;
        token_pos(rope, nbase + r, tl, h, w);
        const float2 cs = rope_cs(rope, reinterpret_cast<const float*>(s_tab), pr, tl, h, w);
        y0 = x0 * cs.x - x1 * cs.y;
        y1 = x0 * cs.y + x1 * cs.x;
      }
      s_kphi[r * D + 2 * pr] = x0;
      s_kphi[r * D + 2 * pr + 1] = x1;
      s_kr[r * D + 2 * pr] = y0;
      s_kr[r * D + 2 * pr + 1] = y1;
      s_v[r * D + 2 * pr] = v0;
      s_v[r * D + 2 * pr + 1] = v1;
    }
    __syncthreads();
    for (int t = 0; t < TT; ++t) {
      float a[R], c[R];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        a[i] = s_kr[t * D + ta * R + i];
        c[i] = s_v[t * D + tc * R + i];
      }
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) acc[i][j] = fmaf(a[i], c[j], acc[i][j]);
      if (tid < D) zacc += s_kphi[t * D + tid];
    }
    __syncthreads();
  }
  if (cur >= 0) flush(cur);
}

// One thread per entry e of the D*(D+1) state of one head. For every segment
// of the head, in order: blk = sum of its partials in CTA order; the apply
// state is run + blk and becomes the new run. run starts at zero, or at the
// carried state (use_state); with commit the final run is written back.
template <int D>
__global__ void __launch_bounds__(256)
reduce_states(const float* __restrict__ partials, Sched sc, float* __restrict__ apply,
              float* __restrict__ stS, float* __restrict__ stz, int use_state, int commit) {
  constexpr int DD = D * D, DD1 = D * (D + 1);
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= DD1) return;
  const int heads = sc.nseg / sc.nblk;
  for (int hh = blockIdx.y; hh < heads; hh += gridDim.y) {
  float run = 0.f;
  if (use_state) run = e < DD ? stS[(long long)hh * DD + e] : stz[(long long)hh * D + (e - DD)];
  // software pipelined over the segments: the first partial of segment b + 1
  // is requested before segment b is summed (same additions, same order)
  const float* base0 = partials + (long long)hh * sc.nblk * sc.maxc * DD1 + e;
  float first = base0[0];
  for (int b = 0; b < sc.nblk; ++b) {
    const int seg = hh * sc.nblk + b;
    const float* base = base0 + (long long)b * sc.maxc * DD1;
    const int np = parts_of(sc, seg);
    const float next = b + 1 < sc.nblk ? base[(long long)sc.maxc * DD1] : 0.f;
    float blk = 0.f + first;
    for (int i = 1; i < np; ++i) blk += base[(long long)i * DD1];
    const float ap = run + blk;
    apply[(long long)seg * DD1 + e] = ap;
    run = ap;
    first = next;
  }
  if (use_state && commit) {
    if (e < DD) stS[(long long)hh * DD + e] = run;
    else stz[(long long)hh * D + (e - DD)] = run;
  }
  }
}

// Apply step on CUDA cores: one CTA per (tile of 32 tokens, segment). S of
// the segment is staged in shared memory; the cos/sin table is read from the
// global copy written by state_partial_simt.
template <int D, typename T>
__global__ void __launch_bounds__(kSimtThreads)
apply_simt(const T* __restrict__ q, const T* __restrict__ g, T* __restrict__ out,
           long long N, Layout lay, Rope rope, int L, int nblk, int tps, int nseg,
           const float* __restrict__ apply,
           const float2* __restrict__ gtab, float eps) {
  constexpr int TT = kSimtTileApply;
  constexpr int DD1 = D * (D + 1);
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* s_S = reinterpret_cast<float*>(smem_raw);  // [D][D]
  float* s_z = s_S + D * D;                          // [D]
  float* s_qphi = s_z + D;                           // [TT][D]
  float* s_qr = s_qphi + TT * D;                     // [TT][D]
  float* s_den = s_qr + TT * D;                      // [TT]
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  if (tile >= tps) return;
  for (int seg = blockIdx.y; seg < nseg; seg += gridDim.y) {
  const int head = seg / nblk, blk = seg - head * nblk;
  const int r0 = tile * TT;
  const int rows = min(TT, L - r0);
  const long long nbase = (long long)blk * L + r0;
  const long long ebase = lay.row(head, nbase, N, D);
  const long long ts = lay.tok_stride(D);

  const float4* src = reinterpret_cast<const float4*>(apply + (long long)seg * DD1);
  for (int i = tid; i < DD1 / 4; i += kSimtThreads) reinterpret_cast<float4*>(s_S)[i] = src[i];
  for (int idx = tid; idx < TT * (D / 2); idx += kSimtThreads) {
    const int r = idx / (D / 2), pr = idx - r * (D / 2);
    float x0 = 0.f, x1 = 0.f;
    if (r < rows) {
      x0 = relu(to_f32(q[ebase + r * ts + 2 * pr]));
      x1 = relu(to_f32(q[ebase + r * ts + 2 * pr + 1]));
    }
    float y0 = x0, y1 = x1;
    if (rope.on && r < rows) {
      int tl, h, w;
      token_pos(rope, nbase + r, tl, h, w);
      const float2 cs = rope_cs(rope, reinterpret_cast<const float*>(gtab), pr, tl, h, w);
      y0 = x0 * cs.x - x1 * cs.y;
      y1 = x0 * cs.y + x1 * cs.x;
    }
    s_qphi[r * D + 2 * pr] = x0;
    s_qphi[r * D + 2 * pr + 1] = x1;
    s_qr[r * D + 2 * pr] = y0;
    s_qr[r * D + 2 * pr + 1] = y1;
  }
  __syncthreads();
  const int warp = tid / 32, lane = tid % 32;
  for (int r = warp; r < TT; r += kSimtThreads / 32) {
    float d = 0.f;
    for (int a = lane; a < D; a += 32) d = fmaf(s_qphi[r * D + a], s_z[a], d);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    if (lane == 0) s_den[r] = d + eps;
  }
  __syncthreads();
  for (int idx = tid; idx < TT * D; idx += kSimtThreads) {
    const int r = idx / D, c = idx - r * D;
    if (r >= rows) continue;
    float num = 0.f;
#pragma unroll 8
    for (int a = 0; a < D; ++a) num = fmaf(s_qr[r * D + a], s_S[a * D + c], num);
    float o = num / s_den[r];
    const long long e = ebase + r * ts + c;
    if (g) o *= sigmoid(to_f32(g[e]));
    out[e] = from_f32<T>(o);
  }
  __syncthreads();
  }
}

// Token-causal apply (Eq. 3 of "Block Linear Attention with Constant-Memory KV
// Cache"): one CTA per chunk of kCausalChunk tokens. With S_<c, z_<c the sums
// over earlier chunks of the head (the inclusive state of the previous chunk,
// written by reduce_states) and P_ij = RoPE(phi q_i) . RoPE(phi k_j),
// Q_ij = phi q_i . phi k_j inside the chunk,
//   out_i = (RoPE(phi q_i) S_<c + sum_{j <= i} P_ij v_j)
//           / (phi q_i . z_<c + sum_{j <= i} Q_ij + eps)   (times sigmoid(g_i)).
template <int D, typename T>
__global__ void __launch_bounds__(kSimtThreads)
apply_causal_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const T* __restrict__ g, T* __restrict__ out, long long N, Layout lay,
                  Rope rope, int nblk,
                  int nseg, const float* __restrict__ apply, const float2* __restrict__ gtab,
                  float eps) {
  constexpr int C = kCausalChunk;
  constexpr int DD1 = D * (D + 1);
  static_assert(C == 32, "the denominator adds one masked weight per lane");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* s_S = reinterpret_cast<float*>(smem_raw);  // [D][D], then z [D]
  float* s_z = s_S + D * D;
  constexpr int KS = D + 1;                          // k row stride: rows j of a warp
  float* s_qphi = s_z + D;                           // [C][D]   fall in distinct banks
  float* s_qr = s_qphi + C * D;
  float* s_kphi = s_qr + C * D;                      // [C][KS]
  float* s_kr = s_kphi + C * KS;
  float* s_v = s_kr + C * KS;                        // [C][D]
  float* s_P = s_v + C * D;                          // [C][C] numerator weights
  float* s_Q = s_P + C * C;                          // [C][C] denominator weights
  float* s_den = s_Q + C * C;                        // [C]
  const int tid = threadIdx.x;
  for (int seg = blockIdx.x; seg < nseg; seg += gridDim.x) {
    const int head = seg / nblk, blk = seg - head * nblk;
    const long long nbase = (long long)blk * C;
    const int rows = (int)min((long long)C, N - nbase);
    const long long ebase = lay.row(head, nbase, N, D);
    const long long ts = lay.tok_stride(D);
    // the state of the chunks before this one (zero for the first)
    if (blk > 0) {
      const float4* src = reinterpret_cast<const float4*>(apply + (long long)(seg - 1) * DD1);
      for (int i = tid; i < DD1 / 4; i += kSimtThreads) reinterpret_cast<float4*>(s_S)[i] = src[i];
    } else {
      for (int i = tid; i < DD1; i += kSimtThreads) s_S[i] = 0.f;
    }
    for (int idx = tid; idx < C * (D / 2); idx += kSimtThreads) {
      const int r = idx / (D / 2), pr = idx - r * (D / 2);
      float qx = 0.f, qy = 0.f, kx = 0.f, ky = 0.f, v0 = 0.f, v1 = 0.f;
      if (r < rows) {
        const long long e = ebase + r * ts + 2 * pr;
        qx = relu(to_f32(q[e]));
        qy = relu(to_f32(q[e + 1]));
        kx = relu(to_f32(k[e]));
        ky = relu(to_f32(k[e + 1]));
        v0 = to_f32(v[e]);
        v1 = to_f32(v[e + 1]);
      }
      float qrx = qx, qry = qy, krx = kx, kry = ky;
      if (rope.on && r < rows) {
        int tl, h, w;
        token_pos(rope, nbase + r, tl, h, w);
        const float2 cs = rope_cs(rope, reinterpret_cast<const float*>(gtab), pr, tl, h, w);
        qrx = qx * cs.x - qy * cs.y;
        qry = qx * cs.y + qy * cs.x;
        krx = kx * cs.x - ky * cs.y;
        kry = kx * cs.y + ky * cs.x;
      }
      const int o = r * D + 2 * pr, ok = r * KS + 2 * pr;
      s_qphi[o] = qx;
      s_qphi[o + 1] = qy;
      s_qr[o] = qrx;
      s_qr[o + 1] = qry;
      s_kphi[ok] = kx;
      s_kphi[ok + 1] = ky;
      s_kr[ok] = krx;
      s_kr[ok + 1] = kry;
      s_v[o] = v0;
      s_v[o + 1] = v1;
    }
    __syncthreads();
    // masked weights inside the chunk (j <= i)
    for (int idx = tid; idx < C * C; idx += kSimtThreads) {
      const int i = idx / C, j = idx - i * C;
      float p = 0.f, qq = 0.f;
      if (j <= i) {
        for (int a = 0; a < D; ++a) {
          p = fmaf(s_qr[i * D + a], s_kr[j * KS + a], p);
          qq = fmaf(s_qphi[i * D + a], s_kphi[j * KS + a], qq);
        }
      }
      s_P[idx] = p;
      s_Q[idx] = qq;
    }
    __syncthreads();
    const int warp = tid / 32, lane = tid % 32;
    for (int r = warp; r < C; r += kSimtThreads / 32) {
      float d = 0.f;
      for (int a = lane; a < D; a += 32) d = fmaf(s_qphi[r * D + a], s_z[a], d);
      d += s_Q[r * C + lane];   // C == 32: one masked weight per lane
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      if (lane == 0) s_den[r] = d + eps;
    }
    __syncthreads();
    for (int idx = tid; idx < C * D; idx += kSimtThreads) {
      const int r = idx / D, c = idx - r * D;
      if (r >= rows) continue;
      float num = 0.f;
#pragma unroll 8
      for (int a = 0; a < D; ++a) num = fmaf(s_qr[r * D + a], s_S[a * D + c], num);
      for (int j = 0; j <= r; ++j) num = fmaf(s_P[r * C + j], s_v[j * D + c], num);
      float o = num / s_den[r];
      const long long e = ebase + r * ts + c;
      if (g) o *= sigmoid(to_f32(g[e]));
      out[e] = from_f32<T>(o);
    }
    __syncthreads();
  }
}

}  // namespace la

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
  int stride[3];     // table entries per position (half, padded so that a
                     // position step is an odd number of 16-byte units)
  int pair_base[3];  // first pair index of each axis
  int tab_off[3];    // first table entry of each axis
  int entries;       // table size in float2
  double theta;
  FastDiv div_hw;    // by Hg * Wg
  FastDiv div_w;     // by Wg
  float rcp_stride[3];  // 1 / stride[a] (exact position recovery for entry < 2^20)
  // theta^(-2m/d) / pi of every pair (pair order) as an unevaluated float sum
  // hi + lo, so that position * frequency / pi is formed to ~2^-48 relative
  float inv_pi_hi[64];
  float inv_pi_lo[64];
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
__device__ __forceinline__ int cta_of_unit_fast(const Sched& s, long long u) {
  return s.fastU ? fdiv(s.divU, (int)((u + 1) * s.G - 1)) : cta_of_unit(s, u);
}

// Number of CTAs (= partial slots) that hold tiles of segment seg.
__device__ __forceinline__ int parts_of(const Sched& s, int seg) {
  const long long ub = (long long)seg * s.tps;
  return cta_of_unit_fast(s, ub + s.tps - 1) - cta_of_unit_fast(s, ub) + 1;
}

__host__ __device__ inline long long slot_index(const Sched& s, int seg, int cta) {
  return (long long)seg * s.maxc + (cta - cta_of_unit(s, (long long)seg * s.tps));
}

// ---- RoPE table ----------------------------------------------------------

// Table stride for an axis with `half` pairs: half rounded up so that one
// position step spans an odd number of 16-byte units (conflict-free loads of
// consecutive positions). Zero-width axes keep stride 0.
__host__ __device__ inline int rope_stride(int half) {
  if (half == 0) return 0;
  int units = (half + 1) / 2;
  if ((units & 1) == 0) ++units;
  return 2 * units;
}

// (cos, sin) of table entry e: the angle pos * theta^(-2m/d) of its axis
// position and pair. With x = angle / pi carried as x_hi + x_lo (the product
// error of x_hi recovered exactly by an FMA), x_hi - 2 rint(x_hi / 2) is exact,
// so the reduced argument r in [-1, 1] is accurate to a few ulp and
// sincospif(r) gives cos(angle), sin(angle) to float precision. Padding
// entries get (1, 0). ih / il are copies of r.inv_pi_hi / r.inv_pi_lo in shared
// memory (lanes read different pairs; a parameter-space read of a per-lane
// index would be serialised).
__device__ inline float2 rope_entry(const Rope& r, const float* ih_tab, const float* il_tab,
                                    int e) {
  int base = 0, stride = r.stride[0], half = r.half[0], pb = 0, toff = r.t_offset;
  float rcp = r.rcp_stride[0];
  if (e >= r.tab_off[2]) {
    base = r.tab_off[2]; stride = r.stride[2]; half = r.half[2]; pb = r.pair_base[2];
    toff = 0; rcp = r.rcp_stride[2];
  } else if (e >= r.tab_off[1]) {
    base = r.tab_off[1]; stride = r.stride[1]; half = r.half[1]; pb = r.pair_base[1];
    toff = 0; rcp = r.rcp_stride[1];
  }
  const int local = e - base;
  const int pos = (int)(((float)local + 0.5f) * rcp);
  const int m = local - pos * stride;
  if (m >= half) return make_float2(1.f, 0.f);
  const float P = (float)(pos + toff);                // exact: positions < 2^24
  const float ih = ih_tab[pb + m], il = il_tab[pb + m];
  const float x_hi = P * ih;
  const float x_lo = fmaf(P, ih, -x_hi) + P * il;
  const float red = (x_hi - 2.f * rintf(0.5f * x_hi)) + x_lo;
  float s, c;
  sincospif(red, &s, &c);
  return make_float2(c, s);
}

// Table entry of pair p (0 .. D/2-1) for a token at local frame tl, row h,
// column w.
__device__ inline int rope_index(const Rope& r, int p, int tl, int h, int w) {
  int ax = p < r.pair_base[1] ? 0 : (p < r.pair_base[2] ? 1 : 2);
  int m = p - r.pair_base[ax];
  int pos = ax == 0 ? tl : (ax == 1 ? h : w);
  return r.tab_off[ax] + pos * r.stride[ax] + m;
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

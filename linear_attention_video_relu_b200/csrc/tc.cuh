// tc.cuh -- tensor-core kernels (tcgen05 MMA, TMEM accumulators, TMA tiles)
// for bf16 I/O with D in {64, 128}.
//
// state_build_tc: per CTA a contiguous range of token tiles. TMA brings the k
//   and v tiles (128-byte swizzle) into a ring of stages; 16 math warps apply
//   phi = ReLU and the 3D RoPE to the k tile in place and sum phi(k) for z;
//   one thread issues tcgen05.mma with A = RoPE(phi k)^T (MN-major) and
//   B = v (MN-major) into an fp32 TMEM accumulator, one per segment (double
//   buffered); 4 epilogue warps copy the finished accumulator and z to the
//   CTA's partial slot. When every head is one segment, the CTA that
//   completes a segment last also sums its partials into the apply image.
// finalize_images: the same reduction for heads of several blocks, with the
//   running sum over blocks.
// apply_tc: per CTA a contiguous range of 128-token tiles. TMA brings q (and
//   the gate logits); 16 math warps write RoPE(phi q) in place and phi(q)
//   into TMEM; one thread issues A = RoPE(phi q) x B = S (K-major, as bf16
//   hi + lo so S keeps ~16 bits) and phi(q) x [z_hi z_lo] into TMEM; the math
//   warps divide by the denominator, apply the gate, round to bf16 and send
//   the tile out (see the apply section for the two output paths).
//
// (SANA-Video paper-graph page, section 3.4: the unnumbered ReLU linear
// attention equation and Eq. 2.) No wait here is unbounded: every mbarrier
// wait gives up after kWaitLimitNs, records the failure in the workspace flag
// and makes the CTA drain its in-flight copies and MMAs and exit.
#pragma once

#include <cuda.h>
#include <mutex>

#include "common.cuh"
#include "linattn.h"
#include "ptx.cuh"

namespace la {

// dynamic shared memory per CTA on sm_100 (227 KB), less 1 KB for the
// kernels' static shared variables
constexpr int kSmemBudget = 227 * 1024 - 1024;
// per CTA when two share an SM (228 KB, 1 KB reserved per CTA, static shared
// variables)
constexpr int kSmemBudgetHalf = 112 * 1024;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

enum : int { kFlagStateTimeout = 1, kFlagApplyTimeout = 2 };

struct TcArgs {
  int D;           // I/O head dim (64, 112 or 128; 112 runs on the 128 kernels)
  long long N;
  int Lq;          // query rows per segment: sc.L, or the query length of a cross-attention
  Rope rope;
  Sched sc;
  long long heads;
  const void *q, *k, *v, *g;
  void* out;
  int* flag;
  float2* gtab;
  float* part;
  float* apply;
  float* stS;
  float* stz;
  int* counters;   // per-segment arrival counters (zero between calls)
  int bnhd, H;     // [B,N,H,D] tensors (else [B,H,N,D]); heads per batch entry
  int fused;       // one segment per head: the state build writes the images
  int use_state, commit, do_apply;
  float eps;
  cudaStream_t stream;
  void* const* events;
};

__host__ __device__ constexpr int tc_state_tile_c(int D) { return D == 128 ? 64 : 128; }
inline int tc_state_tile(int D) { return tc_state_tile_c(D); }
inline int tc_state_ctas_per_sm(int) { return 1; }
constexpr int kApplyTile = 128;

// ---- shared-memory plans (host and device agree on these) -------------------

struct StatePlan {
  int stages;
  uint32_t off_tab, off_pos, off_z, off_bar, off_tmem, total;
};

struct ApplyPlan {
  int stages, sbuf, gst;
  uint32_t off_g, off_S, off_tab, off_pos, off_bar, off_tmem, total;
};

// Bytes of one segment's B-operand image (K-major, 128-byte swizzle): per
// 64-value K half, D rows of S_hi^T then D rows of S_lo^T (bf16); then per K
// half a 16-row block whose row 0 is z_hi, row 1 z_lo and rows 2-15 zero.
__host__ __device__ constexpr uint32_t image_zoff(int D) { return 4u * D * D; }
__host__ __device__ constexpr uint32_t image_bytes(int D) {
  return image_zoff(D) + (uint32_t)(D / 64) * 2048u;
}
__host__ __device__ constexpr uint32_t image_slot(int D) { return (image_bytes(D) + 1023u) / 1024u * 1024u; }

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline StatePlan state_plan(int D, int entries, int stages) {
  StatePlan p;
  const uint32_t stage_bytes = 2u * tc_state_tile_c(D) * D * 2;
  p.stages = stages;
  uint32_t off = stages * stage_bytes;
  p.off_tab = off;
  off = align_up(off + entries * 8u, 32);
  p.off_pos = off;  // per stage: table row offset of each token row, per axis
  off = align_up(off + (entries ? stages * 3u * tc_state_tile_c(D) * 2 : 0), 16);
  p.off_z = off;
  off += 2u * 16 * 8 * 4;  // z of each math warp (8 values), per accumulator buffer
  p.off_bar = align_up(off, 8);
  off = p.off_bar + (3u * stages + 10u) * 8u;
  p.off_tmem = off;
  off += 16;
  p.total = off + 1024;  // slack to align the base to 1024 bytes
  return p;
}

__host__ __device__ inline ApplyPlan apply_plan(int D, int entries, int gate, int stages,
                                                int sbuf, int gst) {
  ApplyPlan p;
  const uint32_t tile = (uint32_t)kApplyTile * D * 2;
  p.stages = stages;
  p.sbuf = sbuf;
  p.gst = gate ? gst : 0;
  uint32_t off = stages * tile;   // q stages
  p.off_g = off;                  // gate tiles: one per stage, or a ring of their own
  off += p.gst * tile;
  p.off_S = align_up(off, 1024);
  off = p.off_S + sbuf * image_slot(D);  // B-operand images, one per S slot
  p.off_tab = align_up(off, 32);
  off = p.off_tab + entries * 8u;
  p.off_pos = align_up(off, 16);
  off = p.off_pos + (entries ? stages * 3u * kApplyTile * 2 : 0);
  p.off_bar = align_up(off, 8);
  off = p.off_bar + (4u * stages + 9u + 2u * p.gst) * 8u;
  p.off_tmem = off;
  off += 16;
  p.total = off + 1024;
  return p;
}

inline int pick_state_stages(int D, int entries) {
  for (int s = 6; s >= 2; --s)
    if (state_plan(D, entries, s).total <= (uint32_t)kSmemBudget) return s;
  return 0;
}

// The apply kernel's output path: at D = 64 the epilogue writes out over the
// q tile and a TMA store sends it (the stage is freed after the store); at
// D = 128 (larger tiles, fewer stages fit) the epilogue stores straight from
// registers, the MMAs free the q stage, and gate tiles have a ring of their own.
__host__ __device__ constexpr bool apply_direct_out(int D) { return D == 128; }

// Two S slots (the next segment's image prefetched while the current one is
// in use) when at least 4 q stages still fit, else one slot and the most
// stages; a gate ring of its own holds two tiles, or one where a large RoPE
// table leaves no room for two (the gate load of the next tile then waits for
// the current tile's epilogue).
inline void pick_apply_plan(int D, int entries, int gate, int* stages, int* sbuf, int* gst,
                            int budget = kSmemBudget) {
  *stages = 0;
  *sbuf = 1;
  *gst = 0;
  auto g = [&](int s) { return gate ? (apply_direct_out(D) ? 2 : s) : 0; };
  for (int s = 8; s >= 4; --s)
    if (apply_plan(D, entries, gate, s, 2, g(s)).total <= (uint32_t)budget) {
      *stages = s;
      *sbuf = 2;
      *gst = g(s);
      return;
    }
  for (int s = 8; s >= 2; --s)
    if (apply_plan(D, entries, gate, s, 1, g(s)).total <= (uint32_t)budget) {
      *stages = s;
      *gst = g(s);
      return;
    }
  if (!gate || !apply_direct_out(D)) return;
  for (int s = 8; s >= 2; --s)
    if (apply_plan(D, entries, gate, s, 1, 1).total <= (uint32_t)budget) {
      *stages = s;
      *gst = 1;
      return;
    }
}

// First tile of CTA c (of g) in the apply kernel's weighted split of u tiles:
// the last `nlate` CTAs weigh 1, the others 2 (nlate = 0 splits evenly). With
// u >= 2 g every CTA gets at least one tile.
__host__ __device__ inline long long apply_tile_start(long long c, int g, int nlate,
                                                      long long u) {
  const long long e = g - nlate;
  const long long w = 2 * (c < e ? c : e) + (c > e ? c - e : 0);
  return w * u / (2 * e + nlate);
}

inline int pick_apply_stages(int D, int entries, int gate) {
  int st, sb, gs;
  pick_apply_plan(D, entries, gate, &st, &sb, &gs);
  return st;
}

// Which calls take the tensor-core kernels: bf16 I/O, D in {64, 128}, and RoPE
// widths that are multiples of 8 (a 16-byte chunk never spans two axes), with
// both kernels' shared memory within budget (gated or not).
// Head dim the tensor-core kernels run at for an I/O head dim: 112-wide rows
// run on the 128 kernels, the tensor maps reading columns 112..127 as zero
// fill and the apply kernel storing only the first 112 columns.
inline int tc_kernel_dim(int D) { return D == 112 ? 128 : D; }

inline bool tc_supported(bool bf16, int D, int rope, int dt, int dh, int dw, int entries) {
  if (!bf16 || (D != 64 && D != 112 && D != 128)) return false;
  if (rope && ((dt % 8) || (dh % 8) || (dw % 8))) return false;
  int e = rope ? entries : 0;
  const int Dk = tc_kernel_dim(D);
  return pick_state_stages(Dk, e) > 0 && pick_apply_stages(Dk, e, 1) > 0;
}

// ---- device helpers ------------------------------------------------------------

// Bounded mbarrier wait: false after kWaitLimitNs (then the flag records it
// and *abort tells the other roles to stop), or as soon as *abort is set.
// Longest sleep of one try_wait; the thread wakes when the phase completes.
constexpr uint32_t kWaitSleepNs = 1000000;

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, int* flag, int code,
                                             volatile int* abort_flag) {
  if (ptx::mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
  const uint64_t t0 = ptx::globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (ptx::mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
    if ((n & 15u) == 0) {
      if (*abort_flag) return false;
      if (ptx::globaltimer() - t0 > kWaitLimitNs) {
        atomicOr(flag, code);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Token position (local frame, row, column) of token n, and a cheap step to
// the token `step` rows further.
struct Pos {
  int tl, h, w;
};

__device__ __forceinline__ Pos pos_of(const Rope& r, int n) {
  Pos p;
  p.tl = fdiv(r.div_hw, n);
  const int rem = n - p.tl * r.div_hw.d;
  p.h = fdiv(r.div_w, rem);
  p.w = rem - p.h * r.Wg;
  return p;
}

__device__ __forceinline__ void pos_advance(const Rope& r, Pos& p, int step) {
  p.w += step;
  while (p.w >= r.Wg) {
    p.w -= r.Wg;
    if (++p.h == r.Hg) {
      p.h = 0;
      ++p.tl;
    }
  }
}

// The rotation pairs of one 16-byte chunk (8 dims) all belong to one axis.
struct ChunkRope {
  int ax;       // axis of the chunk (0 t, 1 h, 2 w)
  int base;     // table entry of (axis, position 0, first pair of the chunk)
  int stride;   // table entries per position on that axis
};

__device__ __forceinline__ ChunkRope chunk_rope(const Rope& r, int chunk) {
  ChunkRope c;
  const int p0 = 4 * chunk;
  c.ax = p0 < r.pair_base[1] ? 0 : (p0 < r.pair_base[2] ? 1 : 2);
  c.stride = r.half[c.ax];
  c.base = r.tab_off[c.ax] + (p0 - r.pair_base[c.ax]);
  return c;
}

// ---- shared pieces of the two kernels --------------------------------------------

constexpr int kMathWarps = 16;
constexpr int kMath = 32 * kMathWarps;  // threads of the math warps (warps 2 .. 17)

// Walks a CTA's contiguous tile range: segment, tile in segment, ring stage
// and phase, all advanced incrementally (no division inside the loops).
struct TileIter {
  int seg, tile, tps;
  int stage, stages;
  uint32_t phase;
  __device__ __forceinline__ void init(long long u0, int tps_, int stages_) {
    tps = tps_;
    seg = (int)(u0 / tps_);
    tile = (int)(u0 - (long long)seg * tps_);
    stages = stages_;
    stage = 0;
    phase = 0;
  }
  __device__ __forceinline__ bool last_of_segment(long long u, long long u1) const {
    return u + 1 == u1 || tile + 1 == tps;
  }
  __device__ __forceinline__ void next() {
    if (++tile == tps) {
      tile = 0;
      ++seg;
    }
    if (++stage == stages) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

// Coordinates of (segment, row) in the 4D tensor maps of q, k, v, gate and
// out. [B,H,N,D] tensors are mapped as {D, L, nseg, 1}: coordinates
// (x, row, seg, 0). [B,N,H,D] tensors as {D, H, L, B * nblk} (strides D, H*D,
// L*H*D elements): coordinates (x, h, row, b * nblk + blk). A box of 64
// columns x rows x one head lands in shared memory in the same order either
// way, and rows past a segment's L read as zero fill in both.
struct SegCoords {
  int bnhd, H, nblk;
  FastDiv div_nblk, div_h;
  __device__ __forceinline__ int3 of(int seg, int row) const {
    if (!bnhd) return make_int3(row, seg, 0);
    const int head = fdiv(div_nblk, seg), blk = seg - head * nblk;
    const int b = fdiv(div_h, head), h = head - b * H;
    return make_int3(h, row, b * nblk + blk);
  }
  // element offset of row r of segment seg (L rows per segment) in an output
  // tensor with rows of ocols values
  __device__ __forceinline__ long long out_row(int seg, int L, int r, int ocols) const {
    if (!bnhd) return ((long long)seg * L + r) * ocols;
    const int head = fdiv(div_nblk, seg), blk = seg - head * nblk;
    const int b = fdiv(div_h, head), h = head - b * H;
    return ((((long long)b * nblk + blk) * L + r) * H + h) * (long long)ocols;
  }
};

// A math warp owns one 16-byte chunk column (8 dims = 4 rotation pairs, all on
// one axis) and its lanes walk consecutive token rows. The TMA warp writes,
// for every row of a tile, the table offset of the row's position on each
// axis (clamped into the table for zero-filled rows past the grid); a chunk
// adds its first pair's index within the axis.
struct ChunkCol {
  int ax, pair_off;
};

__device__ __forceinline__ ChunkCol chunk_col(const Rope& r, int chunk) {
  ChunkCol c;
  const int p0 = 4 * chunk;
  c.ax = p0 < r.pair_base[1] ? 0 : (p0 < r.pair_base[2] ? 1 : 2);
  c.pair_off = p0 - (c.ax == 0 ? 0 : (c.ax == 1 ? r.pair_base[1] : r.pair_base[2]));
  // padding columns past the last rotary pair (a 112-wide head on the 128
  // kernels) hold zeros: any finite cos/sin leaves them zero, so they read
  // the first entries of the t axis
  if (p0 >= r.pair_base[2] + r.half[2]) {
    c.ax = 0;
    c.pair_off = 0;
  }
  return c;
}

// Table row offsets (per axis) of rows [0, rows) of a tile whose first token
// is n0, written by the 32 lanes of the TMA warp.
__device__ __forceinline__ void write_row_offsets(const Rope& r, uint16_t* pos, int rows, int n0,
                                                  int lane) {
  for (int row = lane; row < rows; row += 32) {
    const int n = n0 + row;
    const int tl = fdiv(r.div_hw, n);
    const int rem = n - tl * r.div_hw.d;
    const int h = fdiv(r.div_w, rem);
    const int w = rem - h * r.Wg;
    pos[row] = (uint16_t)(r.tab_off[0] + min(tl, r.T - 1) * r.stride[0]);
    pos[rows + row] = (uint16_t)(r.tab_off[1] + h * r.stride[1]);
    pos[2 * rows + row] = (uint16_t)(r.tab_off[2] + w * r.stride[2]);
  }
}

// phi = ReLU of one 16-byte chunk of bf16 values (4 rotation pairs (x_j, y_j)),
// rotated by the pairs' cos, sin: cs[0] holds the cos of the 4 pairs, cs[1]
// their sin; x' = x cos - y sin, y' = x sin + y cos in fp32, rounded once to
// bf16. xy returns phi as packed float pairs {(x0,x1), (x2,x3), (y0,y1), (y2,y3)},
// m as the 4 bf16x2 words.
template <bool ROPE>
__device__ __forceinline__ uint4 phi_rope(uint4 raw, const float4* cs, uint64_t (&xy)[4],
                                          uint32_t (&m)[4]) {
  const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
  float x[4], y[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m[j]) : "r"(w4[j]), "r"(0u));
    x[j] = ptx::bf16_lo(m[j]);
    y[j] = ptx::bf16_hi(m[j]);
  }
  xy[0] = ptx::f2(x[0], x[1]);
  xy[1] = ptx::f2(x[2], x[3]);
  xy[2] = ptx::f2(y[0], y[1]);
  xy[3] = ptx::f2(y[2], y[3]);
  if (!ROPE) return make_uint4(m[0], m[1], m[2], m[3]);
  const float4 C = cs[0], S = cs[1];
  const uint64_t c01 = ptx::f2(C.x, C.y), c23 = ptx::f2(C.z, C.w);
  const uint64_t s01 = ptx::f2(S.x, S.y), s23 = ptx::f2(S.z, S.w);
  float ox[4], oy[4];
  ptx::f2_split(ptx::sub2(ptx::mul2(xy[0], c01), ptx::mul2(xy[2], s01)), ox[0], ox[1]);
  ptx::f2_split(ptx::sub2(ptx::mul2(xy[1], c23), ptx::mul2(xy[3], s23)), ox[2], ox[3]);
  ptx::f2_split(ptx::fma2(xy[0], s01, ptx::mul2(xy[2], c01)), oy[0], oy[1]);
  ptx::f2_split(ptx::fma2(xy[1], s23, ptx::mul2(xy[3], c23)), oy[2], oy[3]);
  return make_uint4(ptx::pack_bf16x2(ox[0], oy[0]), ptx::pack_bf16x2(ox[1], oy[1]),
                    ptx::pack_bf16x2(ox[2], oy[2]), ptx::pack_bf16x2(ox[3], oy[3]));
}

// Builds the CTA's cos/sin table in shared memory (all math threads), then
// synchronises them.
__device__ __forceinline__ void build_rope_table(const Rope& r, float2* tab, int tt) {
  __shared__ float s_ih[64], s_il[64];
  if (tt < 64) {
    s_ih[tt] = r.inv_pi_hi[tt];
    s_il[tt] = r.inv_pi_lo[tt];
  }
  ptx::bar_sync(1, kMath);
  rope_fill(r, s_ih, s_il, reinterpret_cast<float*>(tab), tt, kMath);
  ptx::bar_sync(1, kMath);
}

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t* v);

template <>
__device__ __forceinline__ void tmem_ld_cols<32>(uint32_t taddr, uint32_t* v) {
  ptx::tmem_ld_32x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(v));
}

template <>
__device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

// ---- image of one segment ----------------------------------------------------------
//
// Partial slots are [D + 1][D] floats: row n < D is column n of S (S[a][n] at
// n * D + a), row D is z. An apply image (layout at image_bytes) is what the
// apply kernel copies into shared memory as its B operands. The 4 values
// a0..a0+3 of row n (< D) go to byte image_offset(n, a0) as hi, D * 128 bytes
// further as lo; those of z to rows 0 (hi) and 1 (lo) of the z block.

template <int D>
__device__ __forceinline__ uint32_t image_offset(int n, int a0) {
  constexpr int SHALF = 2 * D * 128;
  const int ac = a0 >> 3;
  if (n == D) return image_zoff(D) + (ac >> 3) * 2048u + (((ac & 7)) << 4) + ((a0 & 4) << 1);
  return (ac >> 3) * SHALF + n * 128 + (((ac & 7) ^ (n & 7)) << 4) + ((a0 & 4) << 1);
}

template <int D>
__device__ __forceinline__ void store_image4(uint8_t* img, bool zrow, int a0, float4 v) {
  const uint32_t h0 = ptx::pack_bf16x2(v.x, v.y);
  const uint32_t h1 = ptx::pack_bf16x2(v.z, v.w);
  const uint32_t l0 = ptx::pack_bf16x2(v.x - ptx::bf16_lo(h0), v.y - ptx::bf16_hi(h0));
  const uint32_t l1 = ptx::pack_bf16x2(v.z - ptx::bf16_lo(h1), v.w - ptx::bf16_hi(h1));
  *reinterpret_cast<uint2*>(img) = make_uint2(h0, h1);
  if (!zrow) {
    *reinterpret_cast<uint2*>(img + D * 128) = make_uint2(l0, l1);
    return;
  }
  // z block: img is row 0 of chunk ac (unswizzled there); row r holds that
  // chunk at 16-byte position (ac ^ r) & 7 within its 128 bytes
  const int ac = (a0 >> 3) & 7;
  uint8_t* blk = img - ((ac << 4) + ((a0 & 4) << 1));
  const int sub = (a0 & 4) << 1;
  *reinterpret_cast<uint2*>(blk + 128 + (((ac ^ 1) & 7) << 4) + sub) = make_uint2(l0, l1);
#pragma unroll
  for (int r = 2; r < 16; ++r)
    *reinterpret_cast<uint2*>(blk + r * 128 + (((ac ^ r) & 7) << 4) + sub) = make_uint2(0u, 0u);
}

__device__ __forceinline__ float4 add4(float4 x, float4 y) {
  return make_float4(x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w);
}

__device__ __forceinline__ float4 ldcg4(const float* p) {
  return __ldcg(reinterpret_cast<const float4*>(p));
}

// Image (and, when committing, the carried state) of segment seg of a call
// with one segment per head (seg = head): apply = run + blk with blk the
// segment's partials summed in CTA order and run the carried state or zero --
// the fp32 operations of reduce_states. Threads tid, tid + nthr, ... each take
// 4 values of one partial row; loads bypass L1 (other CTAs wrote them).
template <int D>
__device__ void reduce_segment(const float* __restrict__ partials, const Sched& sc, int seg,
                               uint8_t* __restrict__ images, float* __restrict__ stS,
                               float* __restrict__ stz, int use_state, int commit, int tid,
                               int nthr) {
  constexpr int DD = D * D, DD1 = D * (D + 1), QPR = D / 4, ITEMS = (D + 1) * QPR;
  constexpr int BATCH = 8;
  const int np = parts_of(sc, seg);
  const float* base = partials + (long long)seg * sc.maxc * DD1;
  uint8_t* img = images + (long long)seg * image_bytes(D);
  for (int item = tid; item < ITEMS; item += nthr) {
    const int n = item / QPR;
    const int a0 = 4 * (item - n * QPR);
    const bool zrow = n == D;
    const int off = n * D + a0;
    float4 acc = ldcg4(base + off);
    for (int i0 = 1; i0 < np; i0 += BATCH) {
      float4 b[BATCH];
#pragma unroll
      for (int k = 0; k < BATCH; ++k)
        if (i0 + k < np) b[k] = ldcg4(base + (long long)(i0 + k) * DD1 + off);
#pragma unroll
      for (int k = 0; k < BATCH; ++k)
        if (i0 + k < np) acc = add4(acc, b[k]);
    }
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    if (use_state) {
      float r[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        r[e] = zrow ? stz[(long long)seg * D + a0 + e] : stS[(long long)seg * DD + (a0 + e) * D + n];
      run = make_float4(r[0], r[1], r[2], r[3]);
    }
    run = add4(run, acc);
    store_image4<D>(img + image_offset<D>(n, a0), zrow, a0, run);
    if (use_state && commit) {
      const float r[4] = {run.x, run.y, run.z, run.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (zrow) stz[(long long)seg * D + a0 + e] = r[e];
        else stS[(long long)seg * DD + (a0 + e) * D + n] = r[e];
      }
    }
  }
}

// The carried-state values of reduction item `item` (4 consecutive K-values
// a0.. of row n of the transposed state; n = D is z), or zeros.
template <int D>
__device__ __forceinline__ void carried4(const float* gS, const float* gz, int use_state,
                                         int item, float (&r)[4]) {
  constexpr int QPR = D / 4, ITEMS = (D + 1) * QPR;
  const int n = item / QPR;
  const int a0 = 4 * (item - n * QPR);
#pragma unroll
  for (int e = 0; e < 4; ++e) r[e] = 0.f;
  if (use_state && item < ITEMS) {
#pragma unroll
    for (int e = 0; e < 4; ++e) r[e] = n == D ? gz[a0 + e] : gS[(a0 + e) * D + n];
  }
}

// reduce_segment over np partial slots already copied to shared memory
// (slot i at sp + i * D(D + 1)): the same fp32 operations in the same order.
// `first` holds the carried-state values of the thread's first item (loaded
// by the caller while the partials were being copied); each next item's are
// loaded while the thread works on the current one, so the global loads
// overlap instead of costing a round trip per item.
template <int D>
__device__ void reduce_segment_smem(const float* sp, int np, int seg,
                                    uint8_t* __restrict__ images, float* __restrict__ stS,
                                    float* __restrict__ stz, int use_state, int commit, int tid,
                                    int nthr, const float (&first)[4]) {
  constexpr int DD = D * D, DD1 = D * (D + 1), QPR = D / 4, ITEMS = (D + 1) * QPR;
  uint8_t* img = images + (long long)seg * image_bytes(D);
  float* gS = use_state ? stS + (long long)seg * DD : nullptr;
  float* gz = use_state ? stz + (long long)seg * D : nullptr;
  float nxt[4] = {first[0], first[1], first[2], first[3]};
  for (int item = tid; item < ITEMS; item += nthr) {
    const float cur[4] = {nxt[0], nxt[1], nxt[2], nxt[3]};
    carried4<D>(gS, gz, use_state, item + nthr, nxt);
    const int n = item / QPR;
    const int a0 = 4 * (item - n * QPR);
    const bool zrow = n == D;
    const int off = n * D + a0;
    float4 acc = *reinterpret_cast<const float4*>(sp + off);
    for (int i = 1; i < np; ++i)
      acc = add4(acc, *reinterpret_cast<const float4*>(sp + (long long)i * DD1 + off));
    const float4 run = add4(make_float4(cur[0], cur[1], cur[2], cur[3]), acc);
    store_image4<D>(img + image_offset<D>(n, a0), zrow, a0, run);
    if (use_state && commit) {
      const float r[4] = {run.x, run.y, run.z, run.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (zrow) gz[a0 + e] = r[e];
        else gS[(a0 + e) * D + n] = r[e];
      }
    }
  }
}

// The carried state of one segment copied to shared memory transposed, row n
// of T (pitch D + 1 floats) holding column n of S and row D holding z, by
// 4-byte asynchronous copies: consecutive threads read consecutive floats of
// S (the per-item reads of carried4 touch one float per 32-byte sector), the
// pitch spreads their shared-memory writes over all banks, and no register
// holds a value in flight. Complete once the thread's cp_async_wait_all
// returns.
template <int D>
__device__ void load_carried_transposed(const float* __restrict__ gS,
                                        const float* __restrict__ gz, float* T, int tid,
                                        int nthr) {
  constexpr int TP = D + 1;
  const uint32_t t0 = ptx::smem_u32(T);
  for (int i = tid; i < D * D + D; i += nthr) {
    const int a = i / D, n = i - a * D;   // S[a][n], or z[n] for a = D
    ptx::cp_async4(t0 + 4u * (uint32_t)(a < D ? n * TP + a : D * TP + n),
                   a < D ? gS + i : gz + n);
  }
}

// reduce_segment_smem with the carried state in T (load_carried_transposed):
// the same fp32 operations in the same order; when committing, the new state
// goes back into T for store_carried_transposed.
template <int D>
__device__ void reduce_segment_tr(const float* sp, int np, int seg, uint8_t* __restrict__ images,
                                  float* T, int commit, int tid, int nthr) {
  constexpr int DD1 = D * (D + 1), QPR = D / 4, ITEMS = (D + 1) * QPR, TP = D + 1;
  uint8_t* img = images + (long long)seg * image_bytes(D);
  for (int item = tid; item < ITEMS; item += nthr) {
    const int n = item / QPR;
    const int a0 = 4 * (item - n * QPR);
    const int off = n * D + a0;
    float4 acc = *reinterpret_cast<const float4*>(sp + off);
    for (int i = 1; i < np; ++i)
      acc = add4(acc, *reinterpret_cast<const float4*>(sp + (long long)i * DD1 + off));
    float* t = T + n * TP + a0;
    const float4 run = add4(make_float4(t[0], t[1], t[2], t[3]), acc);
    store_image4<D>(img + image_offset<D>(n, a0), n == D, a0, run);
    if (commit) {
      t[0] = run.x;
      t[1] = run.y;
      t[2] = run.z;
      t[3] = run.w;
    }
  }
}

// T back to the carried state in whole float4 rows of S (and z).
template <int D>
__device__ void store_carried_transposed(const float* T, float* __restrict__ gS,
                                         float* __restrict__ gz, int tid, int nthr) {
  constexpr int QPR = D / 4, TP = D + 1;
  for (int item = tid; item < (D + 1) * QPR; item += nthr) {
    const int a = item / QPR;
    const int n0 = 4 * (item - a * QPR);
    if (a < D) {
      *reinterpret_cast<float4*>(gS + a * D + n0) =
          make_float4(T[(n0 + 0) * TP + a], T[(n0 + 1) * TP + a], T[(n0 + 2) * TP + a],
                      T[(n0 + 3) * TP + a]);
    } else {
      const float* t = T + D * TP + n0;
      *reinterpret_cast<float4*>(gz + n0) = make_float4(t[0], t[1], t[2], t[3]);
    }
  }
}

// ---- state build ------------------------------------------------------------------

// warp 0 TMA, warp 1 MMA, warps 2-17 math, warps 18-21 epilogue (one per TMEM
// lane quadrant)
constexpr int kTcThreadsState = 64 + kMath + 128;
constexpr int kTailSegs = 32;   // segments a CTA can leave to its tail

template <int D, bool ROPE>
__global__ void __launch_bounds__(kTcThreadsState, 1)
state_build_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ Rope rope, const __grid_constant__ Sched sc,
               const __grid_constant__ SegCoords scd, int stages, float* __restrict__ partials, float2* __restrict__ gtab, int* flag,
               int* __restrict__ counters, uint8_t* __restrict__ images, float* stS,
               float* stz, int use_state, int commit) {
  constexpr int TT = tc_state_tile_c(D);      // tokens per tile
  constexpr int HALVES = D / 64;              // 64-column (128-byte) halves
  constexpr int HALF_BYTES = TT * 128;        // one half of one tensor's tile
  constexpr int TILE_BYTES = HALVES * HALF_BYTES;
  constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  constexpr int CPR = D / 8;                  // 16-byte chunks per row
  constexpr int WPC = kMathWarps / CPR;       // warps per chunk column
  constexpr int IPW = TT / 32 / WPC;          // 32-row groups per warp and tile
  constexpr int KSTEPS = TT / 16;             // MMAs per tile
  constexpr int DD1 = D * (D + 1);
  constexpr uint32_t IDESC = ptx::idesc_bf16_f32(D, D, 1, 1);
  constexpr uint32_t TMEM_COLS = 2 * D;
  static_assert(WPC >= 1 && IPW * WPC * 32 == TT, "tile must split over the math warps");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  const uint32_t base = align_up(raw_addr, 1024);
  uint8_t* sm = smem_raw + (base - raw_addr);
  const StatePlan P = state_plan(D, ROPE ? rope.entries : 0, stages);
  float2* s_tab = reinterpret_cast<float2*>(sm + P.off_tab);
  uint16_t* s_pos = reinterpret_cast<uint16_t*>(sm + P.off_pos);
  float* s_z = reinterpret_cast<float*>(sm + P.off_z);
  const uint32_t bar0 = base + P.off_bar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto kready_bar = [&](int s) { return bar0 + 8u * (stages + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * stages + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (3 * stages + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (3 * stages + 2 + b); };
  auto zrdy_bar = [&](int b) { return bar0 + 8u * (3 * stages + 4 + b); };
  auto zfree_bar = [&](int b) { return bar0 + 8u * (3 * stages + 6 + b); };
  const uint32_t done_bar = bar0 + 8u * (3 * stages + 8);
  const uint32_t tail_bar = bar0 + 8u * (3 * stages + 9);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + P.off_tmem);
  __shared__ int s_abort;
  __shared__ int s_red;    // segment the epilogue warps reduce at once, or -1
  __shared__ int s_npend;  // segments all warps reduce after the tile loop
  __shared__ int s_pend[kTailSegs];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int cta = blockIdx.x;
  const long long u0 = unit_begin(sc, cta), u1 = unit_begin(sc, cta + 1);

  if (threadIdx.x == 0) {
    s_abort = 0;
    s_npend = 0;
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(kready_bar(s), kMath);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(accf_bar(b), 1);
      ptx::mbar_init(acce_bar(b), 128);
      ptx::mbar_init(zrdy_bar(b), kMathWarps);
      ptx::mbar_init(zfree_bar(b), 128);
    }
    ptx::mbar_init(done_bar, 1);
    ptx::mbar_init(tail_bar, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(s_tmem), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  __syncthreads();
  // Launched early (programmatic dependent launch) behind the previous
  // kernel of the stream: k and v are read, and the workspace is written,
  // only after griddepcontrol.wait (by the TMA warp before its loads, by the
  // math warps before the table goes out; everything else follows the loads).
  // The kernel lets its own dependent (the apply kernel) launch only once it
  // is past that wait: the apply kernel then knows that everything before
  // this kernel in the stream has completed, and reads its q (and gate)
  // tiles before its own wait.

  if (warp == 0) {
    // ---------------- TMA producer (+ row offsets of the RoPE table) ----------------
    ptx::grid_dependency_wait();
    if (lane == 0) ptx::launch_dependents();
    TileIter it;
    it.init(u0, sc.tps, stages);
    long long issued = 0;
    for (long long u = u0; u < u1; ++u, it.next()) {
      int ok = 1;
      if (lane == 0)
        ok = wait_bounded(empty_bar(it.stage), it.phase ^ 1u, flag, kFlagStateTimeout, &s_abort);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (ROPE) {
        const int blk = it.seg - (it.seg / sc.nblk) * sc.nblk;
        write_row_offsets(rope, s_pos + it.stage * 3 * TT, TT, blk * sc.L + it.tile * TT, lane);
        __syncwarp();
      }
      if (lane == 0) {
        const uint32_t kt = base + it.stage * STAGE_BYTES, vt = kt + TILE_BYTES;
        ptx::mbar_expect_tx(full_bar(it.stage), STAGE_BYTES);
        const int3 c = scd.of(it.seg, it.tile * TT);
#pragma unroll
        for (int h = 0; h < HALVES; ++h) {
          ptx::tma_load_4d(kt + h * HALF_BYTES, &tm_k, 64 * h, c.x, c.y, c.z, full_bar(it.stage));
          ptx::tma_load_4d(vt + h * HALF_BYTES, &tm_v, 64 * h, c.x, c.y, c.z, full_bar(it.stage));
        }
      }
      ++issued;
    }
    // drain: every issued copy has landed before the CTA may exit
    if (lane == 0)
      for (long long i = issued - stages < 0 ? 0 : issued - stages; i < issued; ++i)
        wait_bounded(full_bar((int)(i % stages)), (uint32_t)((i / stages) & 1), flag,
                     kFlagStateTimeout, &s_abort);
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t tmem = *s_tmem;
      TileIter it;
      it.init(u0, sc.tps, stages);
      int sidx = 0, first = 1;
      bool ok = wait_bounded(acce_bar(0), 1u, flag, kFlagStateTimeout, &s_abort);
      for (long long u = u0; u < u1 && ok; ++u) {
        if (!wait_bounded(kready_bar(it.stage), it.phase, flag, kFlagStateTimeout, &s_abort))
          break;
        ptx::tc_fence_after();
        const uint32_t kt = base + it.stage * STAGE_BYTES, vt = kt + TILE_BYTES;
        const uint32_t acc = tmem + (uint32_t)((sidx & 1) * D);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const uint64_t a = ptx::smem_desc_sw128(kt + kk * 2048, HALF_BYTES, 1024);
          const uint64_t b = ptx::smem_desc_sw128(vt + kk * 2048, HALF_BYTES, 1024);
          ptx::mma_bf16(acc, a, b, IDESC, (first && kk == 0) ? 0u : 1u);
        }
        ptx::mma_commit(empty_bar(it.stage));
        first = 0;
        if (it.last_of_segment(u, u1)) {
          ptx::mma_commit(accf_bar(sidx & 1));
          ++sidx;
          first = 1;
          if (u + 1 < u1 &&
              !wait_bounded(acce_bar(sidx & 1), (uint32_t)(((sidx >> 1) & 1) ^ 1), flag,
                            kFlagStateTimeout, &s_abort))
            break;
        }
        it.next();
      }
      ptx::mma_commit(done_bar);
      wait_bounded(done_bar, 0, flag, kFlagStateTimeout, &s_abort);
    }
  } else if (warp < 2 + kMathWarps) {
    // ---------------- math warps: ReLU + RoPE, z ----------------
    const int tt = threadIdx.x - 64;
    const int mw = warp - 2;                     // math warp 0..15
    const int c = mw % CPR, rg0 = mw / CPR;      // chunk column, first row group
    const int half = c >> 3, cc = c & 7;
    if (ROPE) {
      build_rope_table(rope, s_tab, tt);
      ptx::grid_dependency_wait();
      const int e0 = (int)((long long)cta * rope.entries / gridDim.x);
      const int e1 = (int)((long long)(cta + 1) * rope.entries / gridDim.x);
      for (int e = e0 + tt; e < e1; e += kMath) gtab[e] = s_tab[e];
    }
    ChunkCol col{};
    if (ROPE) col = chunk_col(rope, c);
    uint64_t z2[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) z2[e] = ptx::f2(0.f, 0.f);
    TileIter it;
    it.init(u0, sc.tps, stages);
    int sidx = 0;
    for (long long u = u0; u < u1; ++u, it.next()) {
      const bool ok = wait_bounded(full_bar(it.stage), it.phase, flag, kFlagStateTimeout,
                                   &s_abort);
      if (ok) {
        const uint32_t kt = base + it.stage * STAGE_BYTES + half * HALF_BYTES;
        const uint16_t* rowoff = s_pos + (it.stage * 3 + col.ax) * TT;
#pragma unroll
        for (int i = 0; i < IPW; ++i) {
          const int r = 32 * (rg0 + WPC * i) + lane;
          const uint32_t addr = kt + r * 128 + ((cc ^ (r & 7)) << 4);
          const uint4 raw = ptx::ld_shared_v4(addr);
          uint64_t f[4];
          uint32_t mw4[4];
          const float4* cs =
              ROPE ? reinterpret_cast<const float4*>(s_tab + rowoff[r] + col.pair_off) : nullptr;
          const uint4 o = phi_rope<ROPE>(raw, cs, f, mw4);
#pragma unroll
          for (int e = 0; e < 4; ++e) z2[e] = ptx::add2(z2[e], f[e]);
          ptx::st_shared_v4(addr, o);
        }
        ptx::fence_proxy_async();
        ptx::mbar_arrive(kready_bar(it.stage));
      }
      if (it.last_of_segment(u, u1)) {
        // hand z over to the epilogue warps: this warp's 32 lanes summed, in
        // the buffer of the segment's accumulator
        const int b = sidx & 1;
        wait_bounded(zfree_bar(b), (uint32_t)(((sidx >> 1) & 1) ^ 1), flag, kFlagStateTimeout,
                     &s_abort);
        // z2 = {(d0,d2), (d4,d6), (d1,d3), (d5,d7)} of the chunk's 8 dims
        float zz[8];
        ptx::f2_split(z2[0], zz[0], zz[2]);
        ptx::f2_split(z2[1], zz[4], zz[6]);
        ptx::f2_split(z2[2], zz[1], zz[3]);
        ptx::f2_split(z2[3], zz[5], zz[7]);
#pragma unroll
        for (int e = 0; e < 4; ++e) z2[e] = ptx::f2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float t = zz[e];
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
          if (lane == 0) s_z[(b * kMathWarps + mw) * 8 + e] = t;
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(zrdy_bar(b));
        ++sidx;
      }
    }
  } else {
    // ---------------- epilogue warps: accumulator and z -> the CTA's partial slot ------
    // slot layout: [D + 1][D] floats, row n < D = column n of S (S[a][n] at
    // n * D + a), row D = z
    const int q = warp & 3;             // TMEM lane quadrant of this warp
    const int te = threadIdx.x - (64 + kMath);
    const uint32_t tmem = *s_tmem;
    // M = 64 keeps rows in lanes 0-15 of each 32-lane quadrant; M = 128 uses
    // all 128 lanes, row = lane.
    const int row = D == 64 ? 16 * q + lane : 32 * q + lane;
    const bool has_row = D == 64 ? lane < 16 : true;
    TileIter it;
    it.init(u0, sc.tps, 1);
    int sidx = 0;
    for (long long u = u0; u < u1; ++u, it.next()) {
      if (!it.last_of_segment(u, u1)) continue;
      const int b = sidx & 1;
      const uint32_t ph = (uint32_t)((sidx >> 1) & 1);
      const bool ready = wait_bounded(accf_bar(b), ph, flag, kFlagStateTimeout, &s_abort) &&
                         wait_bounded(zrdy_bar(b), ph, flag, kFlagStateTimeout, &s_abort);
      ptx::tc_fence_after();
      float* slot = partials + slot_index(sc, it.seg, cta) * DD1;
#pragma unroll 1
      for (int cj = 0; cj < D / 16; ++cj) {
        uint32_t v[16];
        tmem_ld_cols<16>(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * D + 16 * cj), v);
        ptx::tmem_wait_ld();
        if (ready && has_row) {
          // column n of S is row n of the slot: lanes store consecutive a
          float* dst = slot + (size_t)(16 * cj) * D + row;
#pragma unroll
          for (int e = 0; e < 16; ++e) dst[(size_t)e * D] = __uint_as_float(v[e]);
        }
      }
      if (te < D && ready) {
        const int ch = te >> 3, e = te & 7;
        float t = 0.f;
#pragma unroll
        for (int g = 0; g < WPC; ++g) t += s_z[(b * kMathWarps + g * CPR + ch) * 8 + e];
        slot[D * D + te] = t;
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(acce_bar(b));
      ptx::mbar_arrive(zfree_bar(b));
      ++sidx;
      if (counters) {
        // one segment per head: the CTA that completes a segment last turns
        // its partials into the image (all epilogue warps' slot writes are
        // fenced before the arrival is counted) -- after its tile loop with
        // all warps, or here when its list of pending segments is full
        __threadfence();
        const bool all_ready = ptx::bar_all(2, 128, ready);
        if (te == 0) {
          int red = -1;
          if (all_ready) {
            const int old = atomicAdd(counters + it.seg, 1);
            if (old == parts_of(sc, it.seg) - 1) {
              counters[it.seg] = 0;   // every contributor has arrived
              red = it.seg;
            }
          }
          if (red >= 0 && s_npend < kTailSegs) {
            s_pend[s_npend++] = red;  // reduce with all warps after the tile loop
            red = -1;
          }
          s_red = red;
        }
        ptx::bar_sync(2, 128);
        const int red = s_red;
        if (red >= 0) {
          __threadfence();
          reduce_segment<D>(partials, sc, red, images, stS, stz, use_state, commit, te, 128);
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(*s_tmem, TMEM_COLS);
  }
  if (s_npend > 0 && !s_abort) {
    // The drained stage ring (with the tables behind it) takes up to `cap`
    // partial slots: bulk-copy a segment's partials there at once and reduce
    // them from shared memory -- one round trip to L2 for all of them instead
    // of one per row group of each thread.
    constexpr uint32_t SLOT = DD1 * 4;
    constexpr uint32_t TBYTES = (D + 1) * (D + 1) * 4;   // transposed carried state
    const int cap = (int)(P.off_bar / SLOT);
    __threadfence();
    uint32_t tph = 0;
    for (int k = 0; k < s_npend; ++k) {
      const int seg = s_pend[k];
      const int np = parts_of(sc, seg);
      if (np > cap) {
        reduce_segment<D>(partials, sc, seg, images, stS, stz, use_state, commit, threadIdx.x,
                          kTcThreadsState);
        continue;
      }
      if (threadIdx.x == 0) {
        ptx::fence_proxy_async_global();
        ptx::mbar_expect_tx(tail_bar, (uint32_t)np * SLOT);
        for (int i = 0; i < np; ++i)
          ptx::bulk_load(base + (uint32_t)i * SLOT,
                         partials + ((long long)seg * sc.maxc + i) * DD1, SLOT, tail_bar);
      }
      // the carried state goes through shared memory, transposed, behind the
      // partial slots where it fits
      float* gS = use_state ? stS + (long long)seg * D * D : nullptr;
      float* gz = use_state ? stz + (long long)seg * D : nullptr;
      float* T = reinterpret_cast<float*>(sm + (uint32_t)np * SLOT);
      const bool tr = use_state && (uint32_t)np * SLOT + TBYTES <= P.off_bar;
      float first[4];
      if (tr) load_carried_transposed<D>(gS, gz, T, threadIdx.x, kTcThreadsState);
      else carried4<D>(gS, gz, use_state, threadIdx.x, first);
      const bool got = wait_bounded(tail_bar, tph, flag, kFlagStateTimeout, &s_abort);
      if (tr) ptx::cp_async_wait_all();
      if (!__syncthreads_and(got)) break;   // every thread leaves together
      tph ^= 1u;
      if (tr) {
        reduce_segment_tr<D>(reinterpret_cast<const float*>(sm), np, seg, images, T, commit,
                             threadIdx.x, kTcThreadsState);
        if (commit) {
          __syncthreads();
          store_carried_transposed<D>(T, gS, gz, threadIdx.x, kTcThreadsState);
        }
      } else {
        reduce_segment_smem<D>(reinterpret_cast<const float*>(sm), np, seg, images, stS, stz,
                               use_state, commit, threadIdx.x, kTcThreadsState, first);
      }
      __syncthreads();   // before the next segment's copies overwrite the slots
    }
  }
}

// ---- reduction into B-operand images -------------------------------------------------
//
// finalize_images: for every head and every segment of the head in order,
// blk = the segment's partials summed in CTA order, apply = run + blk,
// run = apply, with run starting at zero or at the carried state (written back
// when committing) -- the fp32 operations of reduce_states -- and apply
// written as the segment's image.
//
// Grid (heads, row groups): a thread owns 4 consecutive K-values a0..a0+3 of
// one row n of the column-major partials (n = D is z) of one head, for all of
// the head's segments. The CTA first tabulates the partial count of up to
// kFinSegs segments in shared memory; threads then take the segments in
// batches of BATCH, issuing the loads of the first two partials of every
// segment of a batch before the first add (more than two is rare and loops).
// With few blocks per head (kFinFewBlocks or fewer) the kernel takes batches
// of kFinSmallBatch under a cap of 80 registers per thread (MINB = 6), so that
// the apply kernel's CTAs (608 threads x 64 registers) fit beside two of its
// CTAs on an SM and start while it runs (480p, 7 blocks: 118.8 -> 117.2 us per
// forward on B200); with many blocks, batches of 16 and no cap (fewer rounds
// of loads).

constexpr int kFinThreads = 128;
constexpr int kFinSegs = 1024;
constexpr int kFinFewBlocks = 8;
constexpr int kFinSmallBatch = 4;

template <int D>
__host__ __device__ constexpr int fin_items_per_head() {
  return (D + 1) * (D / 4);
}

template <int D, int BATCH, int MINB>
__global__ void __launch_bounds__(kFinThreads, MINB)
finalize_images(const float* __restrict__ partials, const __grid_constant__ Sched sc,
                uint8_t* __restrict__ images, float* __restrict__ stS,
                float* __restrict__ stz, int use_state, int commit) {
  constexpr int DD = D * D, DD1 = D * (D + 1), QPR = D / 4;
  __shared__ int s_np[kFinSegs];
  ptx::grid_dependency_wait();
  ptx::launch_dependents();
  const int hh = blockIdx.x;
  const int item = blockIdx.y * kFinThreads + threadIdx.x;
  const bool valid = item < fin_items_per_head<D>();
  const int n = item / QPR;
  const int a0 = 4 * (item - n * QPR);
  const bool zrow = n == D;
  const int off = n * D + a0;
  float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
  if (use_state && valid) {
    float r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      r[e] = zrow ? stz[(long long)hh * D + a0 + e] : stS[(long long)hh * DD + (a0 + e) * D + n];
    run = make_float4(r[0], r[1], r[2], r[3]);
  }
  const long long seg0 = (long long)hh * sc.nblk;
  const float* pbase = partials + seg0 * sc.maxc * DD1 + off;
  uint8_t* ibase = images + seg0 * image_bytes(D) + (valid ? image_offset<D>(n, a0) : 0);
  const long long pstride = (long long)sc.maxc * DD1;
  for (int j0 = 0; j0 < sc.nblk; j0 += kFinSegs) {
    const int cnt = min(kFinSegs, sc.nblk - j0);
    for (int jj = threadIdx.x; jj < cnt; jj += kFinThreads)
      s_np[jj] = parts_of(sc, (int)(seg0 + j0 + jj));
    __syncthreads();
    if (valid) {
      for (int jb = 0; jb < cnt; jb += BATCH) {
        float4 b0[BATCH], b1[BATCH];
        int np[BATCH];
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
          np[k] = jb + k < cnt ? s_np[jb + k] : 0;
          const float* p = pbase + (j0 + jb + k) * pstride;
          if (np[k] > 0) b0[k] = __ldg(reinterpret_cast<const float4*>(p));
          if (np[k] > 1) b1[k] = __ldg(reinterpret_cast<const float4*>(p + DD1));
        }
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
          if (np[k] > 0) {
            float4 blk = b0[k];
            if (np[k] > 1) blk = add4(blk, b1[k]);
            const float* p = pbase + (j0 + jb + k) * pstride;
            for (int i = 2; i < np[k]; ++i)
              blk = add4(blk, __ldg(reinterpret_cast<const float4*>(p + (long long)i * DD1)));
            run = add4(run, blk);
            store_image4<D>(ibase + (long long)(j0 + jb + k) * image_bytes(D), zrow, a0, run);
          }
        }
      }
    }
    __syncthreads();
  }
  if (use_state && commit && valid) {
    const float r[4] = {run.x, run.y, run.z, run.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (zrow) stz[(long long)hh * D + a0 + e] = r[e];
      else stS[(long long)hh * DD + (a0 + e) * D + n] = r[e];
    }
  }
}

// ---- apply ---------------------------------------------------------------------------
//
// Per 128-token tile of q (TMA, 128-byte swizzle) the math warps write
// A = RoPE(phi(q)) in place over the tile (bf16: the MMA's A operand in shared
// memory) and phi(q) into tensor memory. The MMA warp accumulates, in
// accumulator buffer b,
//   columns [0, D)      A S_hi + A S_lo        (numerator, S in two bf16 halves)
//   columns [D, D + 16) phi(q) [z_hi, z_lo, 0 ...]   (denominator parts)
// and the epilogue (the math warps, one tile behind their transform) forms
// out = acc / (eps + den) (* sigmoid(g)) as bf16. Output path (apply_direct_out):
// either over the q tile, sent by warp 18 with a TMA store that then frees the
// stage; or stored from registers, with the stage freed by the MMAs and gate
// tiles brought by warp 18 into a ring of their own.

// warp 0 q (+ gate) tiles and images, 1 MMA, 2-17 math, 18 store or gate loads
constexpr int kTcThreadsApply = 96 + kMath;

// At D = 64 without RoPE two apply CTAs share an SM where their plans fit in
// half of its shared memory (4 q stages each instead of 8): the same bytes in
// flight per SM, and twice the math warps per scheduler to hide the per-tile
// chain's shared- and tensor-memory latencies (these variants are compiled
// for 48 registers per thread so that two fit). Cross-attention at 480p x 300
// text tokens: 59.3 -> 54.8 us on B200. With RoPE (one image slot in half the
// memory, the table twice per SM) it was slower, so those keep one CTA.
__host__ __device__ constexpr int apply_min_ctas(int D, bool rope) {
  return D == 64 && !rope ? 2 : 1;
}

__host__ __device__ constexpr uint32_t tmem_cols_pow2(uint32_t n) {
  return n <= 32 ? 32 : (n <= 64 ? 64 : (n <= 128 ? 128 : (n <= 256 ? 256 : 512)));
}

template <int D, bool ROPE, bool GATE, bool LATE>
__global__ void __launch_bounds__(kTcThreadsApply, apply_min_ctas(D, ROPE))
apply_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_g,
         const __grid_constant__ CUtensorMap tm_o, __nv_bfloat16* __restrict__ out, int ocols,
         const __grid_constant__ Rope rope, int L, int nblk,
         const __grid_constant__ SegCoords scd, long long U, int stages, int sbuf, int gst, const uint8_t* __restrict__ images,
         const float2* __restrict__ gtab, float eps, int* flag, int early, int nlate) {
  constexpr int TM = kApplyTile;
  constexpr int HALVES = D / 64;
  constexpr int HALF_BYTES = TM * 128;
  constexpr int TILE_BYTES = HALVES * HALF_BYTES;
  constexpr int SHALF = 2 * D * 128;         // one K-half of an image: S_hi^T, S_lo^T rows
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  constexpr int CPW = CPR / 4;               // chunks per math warp (4 warps per row group)
  constexpr int KSTEPS = D / 16;
  constexpr uint32_t ACC_COLS = D + 16;      // numerator + denominator block
  constexpr uint32_t PHI0 = 2 * ACC_COLS;    // phi(q) buffers: D / 2 columns each
  constexpr uint32_t TMEM_COLS = tmem_cols_pow2(PHI0 + D);
  constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(TM, D, 0, 0);
  constexpr uint32_t IDESC_Z = ptx::idesc_bf16_f32(TM, 16, 0, 0);
  constexpr int EC = D / 4;                  // epilogue columns per thread
  constexpr bool DIRECT = apply_direct_out(D);
  constexpr uint32_t TX = (!DIRECT && GATE ? 2 : 1) * TILE_BYTES;
  static_assert(CPW >= 1 && CPW * 4 == CPR, "chunks must split over 4 warps per row group");
  const int tps = (L + TM - 1) / TM;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  const uint32_t base = align_up(raw_addr, 1024);
  uint8_t* sm = smem_raw + (base - raw_addr);
  const ApplyPlan P = apply_plan(D, ROPE ? rope.entries : 0, GATE ? 1 : 0, stages, sbuf, gst);
  const uint32_t gbase = base + P.off_g;
  constexpr uint32_t IMG = image_bytes(D);
  float2* s_tab = reinterpret_cast<float2*>(sm + P.off_tab);
  uint16_t* s_pos = reinterpret_cast<uint16_t*>(sm + P.off_pos);
  const uint32_t bar0 = base + P.off_bar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto qready_bar = [&](int s) { return bar0 + 8u * (stages + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * stages + s); };
  auto oready_bar = [&](int s) { return bar0 + 8u * (3 * stages + s); };
  const uint32_t bar1 = bar0 + 8u * (4 * stages);
  auto accf_bar = [&](int b) { return bar1 + 8u * b; };
  auto acce_bar = [&](int b) { return bar1 + 8u * (2 + b); };
  auto sfull_bar = [&](int k) { return bar1 + 8u * (4 + k); };
  auto sempty_bar = [&](int k) { return bar1 + 8u * (6 + k); };
  const uint32_t done_bar = bar1 + 8u * 8;
  auto gfull_bar = [&](int k) { return bar1 + 8u * (9 + k); };
  auto gempty_bar = [&](int k) { return bar1 + 8u * (9 + gst + k); };
  auto s_slot = [&](int k) { return base + P.off_S + (uint32_t)k * image_slot(D); };
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + P.off_tmem);
  __shared__ int s_abort;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // tile range: an even split, or (LATE) the last `nlate` CTAs of the grid
  // take half as many tiles as the others (they start last: see the launcher)
  long long u0, u1;
  if constexpr (LATE) {
    u0 = apply_tile_start(blockIdx.x, gridDim.x, nlate, U);
    u1 = apply_tile_start(blockIdx.x + 1, gridDim.x, nlate, U);
  } else {
    u0 = (long long)blockIdx.x * U / gridDim.x;
    u1 = (long long)(blockIdx.x + 1) * U / gridDim.x;
  }

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(qready_bar(s), kMath);
      ptx::mbar_init(empty_bar(s), 1);
      ptx::mbar_init(oready_bar(s), kMath);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(accf_bar(b), 1);
      ptx::mbar_init(acce_bar(b), kMath);
      ptx::mbar_init(sfull_bar(b), 1);
      ptx::mbar_init(sempty_bar(b), 1);
    }
    ptx::mbar_init(done_bar, 1);
    if (DIRECT)
      for (int k = 0; k < gst; ++k) {
        ptx::mbar_init(gfull_bar(k), 1);
        ptx::mbar_init(gempty_bar(k), kMath);
      }
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(s_tmem), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  __syncthreads();
  if (threadIdx.x == 0) ptx::launch_dependents();
  // Launched early (programmatic dependent launch) behind the kernel that
  // writes its images (the state build, or the separate reduction), which
  // lets it launch only once past its own dependency wait: everything before
  // that kernel in the stream -- q and the gate among it -- is complete. So
  // q (and gate) tiles of the first `early` stages may be loaded, and (with a
  // RoPE table built here) transformed, while that kernel still runs; the
  // images, and otherwise the state build's RoPE table, are read only after
  // griddepcontrol.wait.

  if (warp == 0) {
    // ---------------- TMA loads: S images per segment, q (and gate) tiles ----------------
    TileIter it;
    it.init(u0, tps, stages);
    long long issued = 0;
    int cur_seg = -1, ss = -1;
    // q (and gate) tiles into stage it.stage once it is free
    auto load_q = [&](const TileIter& t) -> bool {
      int ok = 1;
      if (lane == 0)
        ok = wait_bounded(empty_bar(t.stage), t.phase ^ 1u, flag, kFlagApplyTimeout, &s_abort);
      if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
      if (ROPE) {
        const int blk = t.seg - (t.seg / nblk) * nblk;
        write_row_offsets(rope, s_pos + t.stage * 3 * TM, TM, blk * L + t.tile * TM, lane);
        __syncwarp();
      }
      if (lane == 0) {
        ptx::mbar_expect_tx(full_bar(t.stage), TX);
        const int3 c = scd.of(t.seg, t.tile * TM);
#pragma unroll
        for (int h = 0; h < HALVES; ++h) {
          ptx::tma_load_4d(base + t.stage * TILE_BYTES + h * HALF_BYTES, &tm_q, 64 * h, c.x,
                           c.y, c.z, full_bar(t.stage));
          if (!DIRECT && GATE)
            ptx::tma_load_4d(gbase + t.stage * TILE_BYTES + h * HALF_BYTES, &tm_g, 64 * h, c.x,
                             c.y, c.z, full_bar(t.stage));
        }
      }
      ++issued;
      return true;
    };
    // `early` stages go out before the wait (the host's choice, by measure)
    const long long pre = u1 - u0 < early ? u1 - u0 : early;
    bool pre_ok = true;
    {
      TileIter ip = it;
      for (long long k = 0; k < pre && pre_ok; ++k, ip.next()) pre_ok = load_q(ip);
    }
    ptx::grid_dependency_wait();
    for (long long u = u0; u < u1 && pre_ok; ++u, it.next()) {
      int ok = 1;
      if (it.seg != cur_seg) {
        // the segment's image into the next slot, once its last user is done
        cur_seg = it.seg;
        ++ss;
        if (lane == 0) {
          const int k = ss % sbuf;
          ok = wait_bounded(sempty_bar(k), (uint32_t)(((ss / sbuf) & 1) ^ 1), flag,
                            kFlagApplyTimeout, &s_abort);
          if (ok) {
            ptx::mbar_expect_tx(sfull_bar(k), IMG);
            ptx::bulk_load(s_slot(k), images + (long long)it.seg * IMG, IMG, sfull_bar(k));
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      if (u - u0 >= pre && !load_q(it)) break;
    }
    if (lane == 0) {
      for (long long i = issued - stages < 0 ? 0 : issued - stages; i < issued; ++i)
        wait_bounded(full_bar((int)(i % stages)), (uint32_t)((i / stages) & 1), flag,
                     kFlagApplyTimeout, &s_abort);
      for (int i = ss - sbuf + 1 < 0 ? 0 : ss - sbuf + 1; i <= ss; ++i)
        wait_bounded(sfull_bar(i % sbuf), (uint32_t)((i / sbuf) & 1), flag, kFlagApplyTimeout,
                     &s_abort);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t tmem = *s_tmem;
      TileIter it;
      it.init(u0, tps, stages);
      int b = 0;
      uint32_t bph = 0;
      int cur_seg = -1, ss = -1;
      uint32_t Sb = 0;
      for (long long u = u0; u < u1; ++u, it.next()) {
        if (it.seg != cur_seg) {
          cur_seg = it.seg;
          ++ss;
          const int k = ss % sbuf;
          if (!wait_bounded(sfull_bar(k), (uint32_t)((ss / sbuf) & 1), flag, kFlagApplyTimeout,
                            &s_abort))
            break;
          Sb = s_slot(k);
        }
        if (!wait_bounded(acce_bar(b), bph ^ 1u, flag, kFlagApplyTimeout, &s_abort)) break;
        if (!wait_bounded(qready_bar(it.stage), it.phase, flag, kFlagApplyTimeout, &s_abort))
          break;
        ptx::tc_fence_after();
        const uint32_t qt = base + it.stage * TILE_BYTES;
        const uint32_t acc = tmem + (uint32_t)b * ACC_COLS;
        const uint32_t phi = tmem + PHI0 + (uint32_t)b * (D / 2);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          // the hi and lo halves of S accumulate into the same columns
          const uint32_t aoff = (kk / 4) * HALF_BYTES + (kk % 4) * 32;
          const uint32_t boff = (kk / 4) * SHALF + (kk % 4) * 32;
          const uint64_t adesc = ptx::smem_desc_sw128(qt + aoff, 16, 1024);
          ptx::mma_bf16(acc, adesc, ptx::smem_desc_sw128(Sb + boff, 16, 1024), IDESC_S,
                        kk == 0 ? 0u : 1u);
          ptx::mma_bf16(acc, adesc, ptx::smem_desc_sw128(Sb + boff + D * 128, 16, 1024),
                        IDESC_S, 1u);
        }
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          // denominator: phi(q) from tensor memory (8 columns per K step)
          const uint32_t zoff = image_zoff(D) + (kk / 4) * 2048 + (kk % 4) * 32;
          ptx::mma_bf16_ta(acc + D, phi + 8u * kk, ptx::smem_desc_sw128(Sb + zoff, 16, 1024),
                           IDESC_Z, kk == 0 ? 0u : 1u);
        }
        ptx::mma_commit(accf_bar(b));
        // once these MMAs have read them, the q stage (with direct output) and,
        // after a segment's last tile, the image slot are free
        if (DIRECT) ptx::mma_commit(empty_bar(it.stage));
        if (it.last_of_segment(u, u1)) ptx::mma_commit(sempty_bar(ss % sbuf));
        if (++b == 2) {
          b = 0;
          bph ^= 1u;
        }
      }
      ptx::mma_commit(done_bar);
      wait_bounded(done_bar, 0, flag, kFlagApplyTimeout, &s_abort);
    }
  } else if (warp == 2 + kMathWarps) {
    if (!DIRECT && lane == 0) {
      // ---------------- TMA stores: out tiles, then free the stage ----------------
      TileIter it;
      it.init(u0, tps, stages);
      for (long long u = u0; u < u1; ++u, it.next()) {
        if (!wait_bounded(oready_bar(it.stage), it.phase, flag, kFlagApplyTimeout, &s_abort))
          break;
        const int3 c = scd.of(it.seg, it.tile * TM);
#pragma unroll
        for (int h = 0; h < HALVES; ++h)
          ptx::tma_store_4d(&tm_o, base + it.stage * TILE_BYTES + h * HALF_BYTES, 64 * h, c.x,
                            c.y, c.z);
        ptx::bulk_commit();
        ptx::bulk_wait_read<0>();
        ptx::mbar_arrive(empty_bar(it.stage));
      }
      ptx::bulk_wait<0>();
    }
    if (DIRECT && GATE && lane == 0) {
      // ---------------- TMA loads of gate tiles into their own ring ----------------
      TileIter it;
      it.init(u0, tps, gst);
      long long issued = 0;
      for (long long u = u0; u < u1; ++u, it.next()) {
        if (!wait_bounded(gempty_bar(it.stage), it.phase ^ 1u, flag, kFlagApplyTimeout,
                          &s_abort))
          break;
        ptx::mbar_expect_tx(gfull_bar(it.stage), TILE_BYTES);
        const int3 c = scd.of(it.seg, it.tile * TM);
#pragma unroll
        for (int h = 0; h < HALVES; ++h)
          ptx::tma_load_4d(gbase + it.stage * TILE_BYTES + h * HALF_BYTES, &tm_g, 64 * h, c.x,
                           c.y, c.z, gfull_bar(it.stage));
        ++issued;
      }
      for (long long i = issued - gst < 0 ? 0 : issued - gst; i < issued; ++i)
        wait_bounded(gfull_bar((int)(i % gst)), (uint32_t)((i / gst) & 1), flag,
                     kFlagApplyTimeout, &s_abort);
    }
  } else {
    // ---------------- math warps: phi(q), RoPE; epilogue ----------------
    // A warp owns the 32 rows of its TMEM lane quadrant and CPW chunk columns.
    const int tt = threadIdx.x - 64;
    const int q4 = warp & 3;                     // TMEM lane quadrant = row group
    const int jw = (warp - 2) >> 2;              // warp within the quadrant, 0..3
    const int row = 32 * q4 + lane;              // tile row of this thread
    const uint32_t lane_bits = (uint32_t)(32 * q4) << 16;
    const int col0 = jw * EC;                    // epilogue columns of this thread
    if (ROPE) {
      // complete before the first lookup: built here where q tiles are
      // transformed before the dependency wait, else copied from the state
      // build's after it
      if (early > 0) {
        build_rope_table(rope, s_tab, tt);
      } else {
        ptx::grid_dependency_wait();
        for (int e = tt; e < rope.entries; e += kMath) s_tab[e] = gtab[e];
        ptx::bar_sync(1, kMath);
      }
    }
    ChunkCol col[CPW];
#pragma unroll
    for (int i = 0; i < CPW; ++i) col[i] = ROPE ? chunk_col(rope, jw * CPW + i) : ChunkCol{};
    const uint32_t tmem = *s_tmem;

    // out rows of tile (seg, tile) in stage s: acc / (eps + den) (* sigmoid(g))
    // as bf16, over the q tile or (direct) from registers to global memory,
    // where rows past the segment's end are not stored
    auto epilogue = [&](int s, int seg, int tile, int eb, uint32_t ebph, int gs, uint32_t gph) {
      const bool ready = wait_bounded(accf_bar(eb), ebph, flag, kFlagApplyTimeout, &s_abort);
      const bool gready = !(DIRECT && GATE) ||
                          wait_bounded(gfull_bar(gs), gph, flag, kFlagApplyTimeout, &s_abort);
      ptx::tc_fence_after();
      const uint32_t lane_base = tmem + lane_bits + (uint32_t)eb * ACC_COLS;
      uint32_t vh[EC], dz[2];
      tmem_ld_cols<EC>(lane_base + col0, vh);
      ptx::tmem_ld_32x32_x2(lane_base + D, dz);
      ptx::tmem_wait_ld();
      const int r = tile * TM + row;
      if (ready && gready && (!DIRECT || r < L)) {
        const float inv = 1.f / (eps + (__uint_as_float(dz[0]) + __uint_as_float(dz[1])));
        const uint64_t inv2 = ptx::f2(inv, inv);
        // rows of ocols values: D, or 112 for a 112-wide head on the 128 kernels
        uint4* dst = reinterpret_cast<uint4*>(out + scd.out_row(seg, L, r, ocols) + col0);
        const uint32_t gt = gbase + (DIRECT ? gs : s) * TILE_BYTES;
        const int h = col0 / 64;
#pragma unroll
        for (int k4 = 0; k4 < EC / 8; ++k4) {
          float o[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint64_t hv = ptx::f2(__uint_as_float(vh[8 * k4 + 2 * e]),
                                        __uint_as_float(vh[8 * k4 + 2 * e + 1]));
            ptx::f2_split(ptx::mul2(hv, inv2), o[2 * e], o[2 * e + 1]);
          }
          const int chunk = (col0 % 64) / 8 + k4;
          const uint32_t off = h * HALF_BYTES + row * 128 + ((chunk ^ (row & 7)) << 4);
          if (GATE) {
            // sigmoid(g) = 1 / (1 + 2^(-g log2 e)) with the approximate
            // exp2 and reciprocal of the special-function unit (a few ulp
            // relative for every g; the output is then rounded to bf16)
            const uint4 gr = ptx::ld_shared_v4(gt + off);
            const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w};
            constexpr float kNegLog2e = -1.4426950408889634f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              o[2 * e] *= ptx::rcp_approx(1.f + ptx::ex2_approx(kNegLog2e * ptx::bf16_lo(gw[e])));
              o[2 * e + 1] *=
                  ptx::rcp_approx(1.f + ptx::ex2_approx(kNegLog2e * ptx::bf16_hi(gw[e])));
            }
          }
          const uint4 ov = make_uint4(ptx::pack_bf16x2(o[0], o[1]), ptx::pack_bf16x2(o[2], o[3]),
                                      ptx::pack_bf16x2(o[4], o[5]), ptx::pack_bf16x2(o[6], o[7]));
          if (DIRECT) {
            if (col0 + 8 * k4 < ocols) dst[k4] = ov;
          } else {
            ptx::st_shared_v4(base + s * TILE_BYTES + off, ov);
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(acce_bar(eb));
      if (DIRECT && GATE) ptx::mbar_arrive(gempty_bar(gs));
      if (!DIRECT) {
        ptx::fence_proxy_async();
        ptx::mbar_arrive(oready_bar(s));
      }
    };

    int pend_stage = -1, pend_seg = 0, pend_tile = 0, pend_b = 0, pend_g = 0;
    uint32_t pend_bph = 0, pend_gph = 0;
    int b = 0;
    uint32_t bph = 0;
    int gslot = 0;
    uint32_t gphase = 0;
    TileIter it;
    it.init(u0, tps, stages);
    for (long long u = u0; u < u1; ++u, it.next()) {
      const bool ok = wait_bounded(full_bar(it.stage), it.phase, flag, kFlagApplyTimeout,
                                   &s_abort);
      if (ok) {
        // A = RoPE(phi q) in place; phi q into the tensor memory of buffer b,
        // whose last reader (the MMAs of two tiles ago) the epilogue of the
        // previous tile has waited for
        const uint32_t tphi = tmem + lane_bits + PHI0 + (uint32_t)b * (D / 2);
#pragma unroll
        for (int i = 0; i < CPW; ++i) {
          const int c = jw * CPW + i;
          const uint32_t addr = base + it.stage * TILE_BYTES + (c >> 3) * HALF_BYTES +
                                row * 128 + (((c & 7) ^ (row & 7)) << 4);
          const uint4 raw = ptx::ld_shared_v4(addr);
          uint64_t xy[4];
          uint32_t m[4];
          const float4* cs =
              ROPE ? reinterpret_cast<const float4*>(
                         s_tab + s_pos[(it.stage * 3 + col[i].ax) * TM + row] + col[i].pair_off)
                   : nullptr;
          const uint4 o = phi_rope<ROPE>(raw, cs, xy, m);
          ptx::st_shared_v4(addr, o);
          ptx::tmem_st_32x32_x4(tphi + 4u * c, m);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::fence_proxy_async();
        ptx::mbar_arrive(qready_bar(it.stage));
      }
      if (pend_stage >= 0)
        epilogue(pend_stage, pend_seg, pend_tile, pend_b, pend_bph, pend_g, pend_gph);
      pend_stage = it.stage;
      pend_seg = it.seg;
      pend_tile = it.tile;
      pend_b = b;
      pend_bph = bph;
      pend_g = gslot;
      pend_gph = gphase;
      if (++b == 2) {
        b = 0;
        bph ^= 1u;
      }
      if (DIRECT && GATE && ++gslot == gst) {
        gslot = 0;
        gphase ^= 1u;
      }
    }
    if (pend_stage >= 0)
      epilogue(pend_stage, pend_seg, pend_tile, pend_b, pend_bph, pend_g, pend_gph);
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(*s_tmem, TMEM_COLS);
  }
}

// ---- host launcher ---------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// [nseg][L][D] bf16 view of a [B,H,N,D] tensor; box = 64 columns x rows x 1.
// 4D map of a bf16 tensor of rows D values wide, cut into segments of L rows
// (see SegCoords): {D, L, nseg, 1} for [B,H,N,D], {D, H, L, B * nblk} for
// [B,N,H,D]; box 64 columns x `rows` rows of one segment.
inline bool make_map(CUtensorMap* m, const void* ptr, int D, int L, int nseg, int rows,
                     const SegCoords& sc) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t row = (cuuint64_t)D * 2;   // bytes of one row
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4] = {64, 1, 1, 1};
  if (!sc.bnhd) {
    dims[0] = (cuuint64_t)D; dims[1] = (cuuint64_t)L; dims[2] = (cuuint64_t)nseg; dims[3] = 1;
    strides[0] = row;
    strides[1] = row * (cuuint64_t)L;
    strides[2] = row * (cuuint64_t)L * (cuuint64_t)nseg;
    box[1] = (cuuint32_t)rows;
  } else {
    const cuuint64_t H = (cuuint64_t)sc.H;
    dims[0] = (cuuint64_t)D; dims[1] = H; dims[2] = (cuuint64_t)L;
    dims[3] = (cuuint64_t)nseg / H;            // B * nblk
    strides[0] = row;
    strides[1] = row * H;
    strides[2] = row * H * (cuuint64_t)L;
    box[2] = (cuuint32_t)rows;
  }
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

inline la_status tc_mark(const TcArgs& a, int i) {
  if (!a.events || !a.events[i]) return LA_OK;
  if (cudaEventRecord(static_cast<cudaEvent_t>(a.events[i]), a.stream) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  return LA_OK;
}

inline la_status tc_check_launch() {
  if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
  return LA_OK;
}

// Launch with programmatic stream serialisation: the kernel may begin while
// the previous kernel on the stream is finishing and must call
// griddepcontrol.wait before it touches that kernel's results.
template <typename... KArgs, typename... Args>
inline la_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  return LA_OK;
}

// The tensor-core kernels whose shared-memory attributes are set, as one bit
// per device (ordinals below 64) for each kernel: a call then costs no
// attribute calls. Guarded by a mutex, so calls stay re-entrant; a context
// reset (cudaDeviceReset) drops the attributes but not this record, and the
// next launch then fails with LA_ERR_CUDA.
class AttrRegistry {
 public:
  bool has(const void* fn, int dev) {
    std::lock_guard<std::mutex> g(mu_);
    for (int i = 0; i < n_; ++i)
      if (fn_[i] == fn) return (mask_[i] >> dev) & 1u;
    return false;
  }
  void add(const void* fn, int dev) {
    std::lock_guard<std::mutex> g(mu_);
    for (int i = 0; i < n_; ++i)
      if (fn_[i] == fn) {
        mask_[i] |= 1ull << dev;
        return;
      }
    if (n_ < kMax) {
      fn_[n_] = fn;
      mask_[n_++] = 1ull << dev;
    }
  }

 private:
  static constexpr int kMax = 64;
  std::mutex mu_;
  const void* fn_[kMax] = {};
  uint64_t mask_[kMax] = {};
  int n_ = 0;
};

inline AttrRegistry& attr_registry() {
  static AttrRegistry r;
  return r;
}

// Every plan of a tensor-core kernel fits kSmemBudget, so the dynamic
// shared-memory limit is set to that once per kernel and device (the launch's
// own size decides how many CTAs share an SM).
template <typename K>
inline la_status tc_smem_attr(K kernel, uint32_t bytes) {
  if (bytes > (uint32_t)kSmemBudget) return LA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  const void* fn = reinterpret_cast<const void*>(kernel);
  const bool record = dev >= 0 && dev < 64;
  if (record && attr_registry().has(fn, dev)) return LA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget) !=
      cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_UNSUPPORTED;
  }
  // the whole unified L1/shared array as shared memory, so that two apply
  // CTAs of half the budget can share an SM (a hint; nothing else relies on it)
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    cudaGetLastError();
  if (record) attr_registry().add(fn, dev);
  return LA_OK;
}

template <int D>
la_status tc_run_d(const TcArgs& a, int sms) {
  const int entries = a.rope.on ? a.rope.entries : 0;
  const Sched& sc = a.sc;
  CUtensorMap mk, mv, mq, mg, mo;
  SegCoords scd;
  scd.bnhd = a.bnhd;
  scd.H = a.H > 0 ? a.H : 1;
  scd.nblk = sc.nblk;
  scd.div_nblk = make_fastdiv(sc.nblk);
  scd.div_h = make_fastdiv(scd.H);
  // tensor maps over the I/O rows (a.D wide); columns past a.D read as zeros
  if (!make_map(&mk, a.k, a.D, sc.L, sc.nseg, tc_state_tile_c(D), scd) ||
      !make_map(&mv, a.v, a.D, sc.L, sc.nseg, tc_state_tile_c(D), scd))
    return LA_ERR_CUDA;
  la_status st;
  const int s1 = pick_state_stages(D, entries);
  const StatePlan p1 = state_plan(D, entries, s1);
  auto k1 = a.rope.on ? state_build_tc<D, true> : state_build_tc<D, false>;
  if ((st = tc_smem_attr(k1, p1.total)) != LA_OK) return st;
  if ((st = tc_mark(a, 0)) != LA_OK) return st;
  uint8_t* images = reinterpret_cast<uint8_t*>(a.apply);
  st = launch_pdl(k1, dim3(sc.G), dim3(kTcThreadsState), p1.total, a.stream, mk, mv, a.rope,
                  sc, scd, s1, a.part, a.gtab, a.flag, a.fused ? a.counters : nullptr, images,
                  a.stS, a.stz, a.use_state, a.commit);
  if (st != LA_OK) return st;
  if ((st = tc_mark(a, 1)) != LA_OK) return st;
  if (!a.fused) {
    // the reduction and the apply kernel are launched programmatically
    // dependent: they start early and wait in griddepcontrol.wait
    const dim3 grid((unsigned)a.heads, (fin_items_per_head<D>() + kFinThreads - 1) / kFinThreads);
    st = sc.nblk <= kFinFewBlocks
             ? launch_pdl(finalize_images<D, kFinSmallBatch, 6>, grid, dim3(kFinThreads), 0,
                          a.stream, (const float*)a.part, sc, images, a.stS, a.stz,
                          a.use_state, a.commit)
             : launch_pdl(finalize_images<D, 16, 1>, grid, dim3(kFinThreads), 0, a.stream,
                          (const float*)a.part, sc, images, a.stS, a.stz, a.use_state,
                          a.commit);
    if (st != LA_OK) return st;
  }
  if ((st = tc_mark(a, 2)) != LA_OK) return st;
  if (!a.do_apply) return LA_OK;

  const bool gate = a.g != nullptr;
  if (!make_map(&mq, a.q, a.D, a.Lq, sc.nseg, kApplyTile, scd) ||
      !make_map(&mo, a.out, a.D, a.Lq, sc.nseg, kApplyTile, scd) ||
      !make_map(&mg, gate ? a.g : a.q, a.D, a.Lq, sc.nseg, kApplyTile, scd))
    return LA_ERR_CUDA;
  int s3 = 0, sb3 = 1, gs3 = 0, cps = 1;   // cps: apply CTAs per SM
  if (apply_min_ctas(D, a.rope.on != 0) == 2) {
    pick_apply_plan(D, entries, gate ? 1 : 0, &s3, &sb3, &gs3, kSmemBudgetHalf);
    if (s3 >= 3) cps = 2;
  }
  if (cps == 1) pick_apply_plan(D, entries, gate ? 1 : 0, &s3, &sb3, &gs3);
  const ApplyPlan p3 = apply_plan(D, entries, gate ? 1 : 0, s3, sb3, gs3);
  const long long U3 = (long long)sc.nseg * ((a.Lq + kApplyTile - 1) / kApplyTile);
  // q (and gate) stages the apply kernel loads before its dependency wait,
  // by measure on B200: two behind a state build that reduces its own
  // segments, at D = 128, without RoPE, and in small calls (up to 8 tiles
  // per SM, e.g. block steps, where the apply's start is most of its time);
  // none on large D = 64 RoPE calls and behind the separate reduction kernel,
  // where the early traffic slowed the reductions (L2-latency bound) more
  // than it saved
  const int early = a.fused && (D == 128 || !a.rope.on || U3 <= 8LL * sms) ? 2 : 0;
  const int G3 = (int)(U3 < (long long)sms * cps ? U3 : (long long)sms * cps);
  // Behind a state build that reduces its own segments, the apply CTAs are
  // placed in index order on the SMs the state-build CTAs leave, and those
  // that reduce leave last: in a small call (a few tiles per CTA) the last
  // CTAs would start too late to finish with the rest, so the last
  // (one per segment) take half as many tiles
  const int nlate = a.fused && U3 <= 8LL * sms && U3 >= 2LL * G3 && 4 * sc.nseg <= G3
                        ? sc.nseg : 0;
  // (a separate instantiation, so that the even split compiles as before)
  auto k3 = nlate > 0
                ? (a.rope.on ? (gate ? apply_tc<D, true, true, true> : apply_tc<D, true, false, true>)
                             : (gate ? apply_tc<D, false, true, true>
                                     : apply_tc<D, false, false, true>))
                : (a.rope.on ? (gate ? apply_tc<D, true, true, false>
                                     : apply_tc<D, true, false, false>)
                             : (gate ? apply_tc<D, false, true, false>
                                     : apply_tc<D, false, false, false>));
  if ((st = tc_smem_attr(k3, p3.total)) != LA_OK) return st;
  st = launch_pdl(k3, dim3(G3), dim3(kTcThreadsApply), p3.total, a.stream, mq, mg, mo,
                  static_cast<__nv_bfloat16*>(a.out), a.D, a.rope, a.Lq, sc.nblk, scd, U3, s3,
                  sb3, gs3,
                  reinterpret_cast<const uint8_t*>(a.apply), (const float2*)a.gtab, a.eps,
                  a.flag, early, nlate);
  if (st != LA_OK) return st;
  return tc_mark(a, 3);
}

inline la_status tc_run(const TcArgs& a, int sms) {
  if (a.D == 64) return tc_run_d<64>(a, sms);
  if (a.D == 112 || a.D == 128) return tc_run_d<128>(a, sms);
  return LA_ERR_UNSUPPORTED;
}

}  // namespace la

// causal.cuh -- per-token causal ReLU linear attention on the tensor cores
// (bf16 I/O, D = 64): out_i uses the sums over tokens 0..i of its head, the
// causal form of "Block Linear Attention with Constant-Memory KV Cache"
// (Eq. 3, SANA-Video paper-graph page), with RoPE on phi in the numerator
// only as in Eq. 2.
//
// Two launches. The state build (state_build_tc, one segment per head, no
// reduction) writes per (head, CTA) the partial S, z of the CTA's contiguous
// range of 128-token tiles. causal_tc then gives every CTA the same range:
// it starts from the sum of the partials of the earlier CTAs of its first
// head (in CTA order, so the result is deterministic; zero for a CTA that
// starts a head) and walks its tiles in order, carrying the state. Per
// 128-token chunk c, with A = RoPE(phi Q_c), Kr = RoPE(phi K_c):
//   P      = A Kr^T                     tensor cores, fp32 in tensor memory
//   P_m    = P with P_ij = 0 for j > i  math warps, bf16 back into tensor
//                                        memory (the A operand of P_m V)
//   num    = A S_<c + P_m V_c           tensor cores (S_<c as bf16 hi + lo)
//   S_<c+1 = S_<c + Kr^T V_c            tensor cores, fp32 in tensor memory
//   den_i  = phi q_i . (z_<c + sum_{j <= i in c} phi k_j) + eps
//            math warps: a running key sum down the chunk's rows (warp
//            scans), fp32
//   out_i  = num_i / den_i (* sigmoid(g_i)), rounded to bf16.
// After each chunk the math warps turn the fp32 state into the bf16 hi/lo
// image the next chunk's A S_<c reads.
//
// Roles: warp 0 TMA (q, k, v tiles of a chunk into one stage), warp 1 MMA
// (one thread), warps 2-17 math. Every mbarrier wait is bounded.
#pragma once

#include "tc.cuh"

namespace la {

constexpr int kCausalTcThreads = 64 + kMath;
constexpr uint32_t kCTile = 128 * 64 * 2;   // one 128 x 64 bf16 tile (16 KB)

struct CausalPlan {
  int stages;
  uint32_t off_simg, off_tab, off_pos, off_den, off_wtot, off_zs, off_bar, off_tmem, total;
};

// barriers: full, kready, empty per stage; pfull, pm, sfull, simg, numfull[2],
// numfree[2], done
__host__ __device__ constexpr int causal_nbar(int stages) { return 3 * stages + 9; }

__host__ __device__ inline CausalPlan causal_plan(int entries, int stages) {
  CausalPlan p;
  p.stages = stages;
  uint32_t off = stages * 3u * kCTile;         // q, k, v tiles per stage
  p.off_simg = off;
  off += 2u * 2u * 64u * 128u;                 // two S images (hi rows, lo rows)
  p.off_tab = off;
  off = align_up(off + entries * 8u, 16);
  p.off_pos = off;
  off = align_up(off + (entries ? stages * 3u * 128u * 2u : 0u), 16);
  p.off_den = off;
  off += 3u * 8u * 128u * 4u;                  // denominator parts [chunk % 3][col][row]
  p.off_wtot = off;
  off += 2u * 2u * 8u * 8u * 4u;               // key-sum totals [buf][row half][col][8]
  p.off_zs = off;
  off += 64u * 4u;                             // z of the start state
  p.off_bar = align_up(off, 8);
  off = p.off_bar + causal_nbar(stages) * 8u;
  p.off_tmem = off;
  off += 16;
  p.total = off + 1024;
  return p;
}

inline int pick_causal_stages(int entries) {
  for (int s = 3; s >= 2; --s)
    if (causal_plan(entries, s).total <= (uint32_t)kSmemBudget) return s;
  return 0;
}

__device__ __forceinline__ void tmem_st_32x32_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// S image: the B operand of A S in MN-major form (64 rows a = K, 64 values d
// = N per 128-byte row, 128-byte swizzle), hi rows then lo rows 8 KB further
// -- the layout of the tensor-memory rows of S, so a thread owning row a
// writes its values with 16-byte stores. Byte offset of the 16-byte chunk
// holding d = 8 cd .. 8 cd + 7 of row a:
__device__ __forceinline__ uint32_t simg_chunk(int a, int cd) {
  return (uint32_t)(a * 128 + (((cd ^ (a & 7)) & 7) << 4));
}

// The 8 fp32 values v[0..7] as bf16 hi + lo (v - hi) 16-byte chunks.
__device__ __forceinline__ void split_hilo8(const uint32_t* v, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float x = __uint_as_float(v[2 * e]), y = __uint_as_float(v[2 * e + 1]);
    h[e] = ptx::pack_bf16x2(x, y);
    l[e] = ptx::pack_bf16x2(x - ptx::bf16_lo(h[e]), y - ptx::bf16_hi(h[e]));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Warp-wide inclusive prefix sum over the lanes of 8 values.
__device__ __forceinline__ void warp_scan8(float (&v)[8], int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float t = __shfl_up_sync(0xffffffffu, v[e], o);
      if (lane >= o) v[e] += t;
    }
  }
}

template <bool ROPE, bool GATE>
__global__ void __launch_bounds__(kCausalTcThreads, 1)
causal_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ Rope rope,
          const __grid_constant__ Sched sc, const __grid_constant__ SegCoords scd, int stages,
          const float* __restrict__ partials, const float2* __restrict__ gtab,
          const __nv_bfloat16* __restrict__ g, __nv_bfloat16* __restrict__ out, float eps,
          int* flag) {
  constexpr int D = 64;
  constexpr int TM = 128;                       // chunk rows (= the state build's tile)
  constexpr int DD1 = D * (D + 1);
  constexpr uint32_t HALF = TM * 128;           // one 64-column half of a 128-row tile
  constexpr uint32_t IDESC_P = ptx::idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(64, 64, 1, 1);
  constexpr uint32_t IDESC_N2 = ptx::idesc_bf16_f32(128, 64, 0, 1);
  constexpr uint32_t IDESC_N3 = ptx::idesc_bf16_f32(128, 64, 0, 1);
  // tensor memory columns
  constexpr uint32_t TP = 0;                    // P: 128 lanes x 128 columns
  constexpr uint32_t TNUM = 128;                // two 64-column numerator buffers
  constexpr uint32_t TS = 256;                  // S: M = 64 (lanes 0-15 of each quadrant)
  constexpr uint32_t TPM = 320;                 // P_m: bf16 pairs, 64 columns
  constexpr uint32_t TMEM_COLS = 512;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  const uint32_t base = align_up(raw_addr, 1024);
  uint8_t* sm = smem_raw + (base - raw_addr);
  const CausalPlan P = causal_plan(ROPE ? rope.entries : 0, stages);
  float2* s_tab = reinterpret_cast<float2*>(sm + P.off_tab);
  uint16_t* s_pos = reinterpret_cast<uint16_t*>(sm + P.off_pos);
  float* s_den = reinterpret_cast<float*>(sm + P.off_den);
  float* s_wtot = reinterpret_cast<float*>(sm + P.off_wtot);
  float* s_zs = reinterpret_cast<float*>(sm + P.off_zs);
  const uint32_t simg_base = base + P.off_simg;
  const uint32_t bar0 = base + P.off_bar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto kready_bar = [&](int s) { return bar0 + 8u * (stages + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * stages + s); };
  const uint32_t pfull_bar = bar0 + 8u * (3 * stages);
  const uint32_t pm_bar = bar0 + 8u * (3 * stages + 1);
  const uint32_t sfull_bar = bar0 + 8u * (3 * stages + 2);
  const uint32_t simg_bar = bar0 + 8u * (3 * stages + 3);
  auto numfull_bar = [&](int b) { return bar0 + 8u * (3 * stages + 4 + b); };
  auto numfree_bar = [&](int b) { return bar0 + 8u * (3 * stages + 6 + b); };
  const uint32_t done_bar = bar0 + 8u * (3 * stages + 8);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + P.off_tmem);
  __shared__ int s_abort;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int cta = blockIdx.x;
  const long long u0 = unit_begin(sc, cta), u1 = unit_begin(sc, cta + 1);
  const int L = sc.L;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(kready_bar(s), kMath);
      ptx::mbar_init(empty_bar(s), 1);
    }
    ptx::mbar_init(pfull_bar, 1);
    ptx::mbar_init(pm_bar, kMath);
    ptx::mbar_init(sfull_bar, 1);
    ptx::mbar_init(simg_bar, kMath);
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(numfull_bar(b), 1);
      ptx::mbar_init(numfree_bar(b), kMath);
    }
    ptx::mbar_init(done_bar, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(s_tmem), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  __syncthreads();
  if (threadIdx.x == 0) ptx::launch_dependents();
  // launched early behind the state build (programmatic dependent launch):
  // its partials and table are read only after griddepcontrol.wait
  ptx::grid_dependency_wait();

  if (warp == 0) {
    // ---------------- TMA: q, k, v tiles of each chunk ----------------
    TileIter it;
    it.init(u0, sc.tps, stages);
    long long issued = 0;
    for (long long u = u0; u < u1; ++u, it.next()) {
      int ok = 1;
      if (lane == 0)
        ok = wait_bounded(empty_bar(it.stage), it.phase ^ 1u, flag, kFlagApplyTimeout, &s_abort);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (ROPE) {
        write_row_offsets(rope, s_pos + it.stage * 3 * TM, TM, it.tile * TM, lane);
        __syncwarp();
      }
      if (lane == 0) {
        const uint32_t st = base + it.stage * 3u * kCTile;
        ptx::mbar_expect_tx(full_bar(it.stage), 3u * kCTile);
        const int3 c = scd.of(it.seg, it.tile * TM);
        ptx::tma_load_4d(st, &tm_q, 0, c.x, c.y, c.z, full_bar(it.stage));
        ptx::tma_load_4d(st + kCTile, &tm_k, 0, c.x, c.y, c.z, full_bar(it.stage));
        ptx::tma_load_4d(st + 2u * kCTile, &tm_v, 0, c.x, c.y, c.z, full_bar(it.stage));
      }
      ++issued;
    }
    if (lane == 0)
      for (long long i = issued - stages < 0 ? 0 : issued - stages; i < issued; ++i)
        wait_bounded(full_bar((int)(i % stages)), (uint32_t)((i / stages) & 1), flag,
                     kFlagApplyTimeout, &s_abort);
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t tmem = *s_tmem;
      TileIter it;
      it.init(u0, sc.tps, stages);
      long long c = 0;   // chunk count of this CTA
      for (long long u = u0; u < u1; ++u, ++c, it.next()) {
        const int b = (int)(c & 1);
        const uint32_t cph = (uint32_t)(c & 1);
        if (!wait_bounded(kready_bar(it.stage), it.phase, flag, kFlagApplyTimeout, &s_abort)) break;
        ptx::tc_fence_after();
        const uint32_t qt = base + it.stage * 3u * kCTile, kt = qt + kCTile, vt = kt + kCTile;
        // P = A Kr^T (the math warps have read the previous chunk's P)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::mma_bf16(tmem + TP, ptx::smem_desc_sw128(qt + kk * 32, 16, 1024),
                        ptx::smem_desc_sw128(kt + kk * 32, 16, 1024), IDESC_P, kk ? 1u : 0u);
        ptx::mma_commit(pfull_bar);
        // S += Kr^T V once the math warps have imaged (and, at a head's
        // start, reset) the state of the previous chunk
        if (!wait_bounded(simg_bar, cph, flag, kFlagApplyTimeout, &s_abort)) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16(tmem + TS, ptx::smem_desc_sw128(kt + kk * 2048, HALF, 1024),
                        ptx::smem_desc_sw128(vt + kk * 2048, HALF, 1024), IDESC_S, 1u);
        ptx::mma_commit(sfull_bar);
        // num = A S_<c (image of the previous chunk's state) + P_m V
        if (!wait_bounded(numfree_bar(b), (uint32_t)(((c >> 1) & 1) ^ 1), flag, kFlagApplyTimeout,
                          &s_abort))
          break;
        const uint32_t simg = simg_base + (uint32_t)((c + 1) & 1) * 16384u;
        const uint32_t acc = tmem + TNUM + (uint32_t)b * 64u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t adesc = ptx::smem_desc_sw128(qt + kk * 32, 16, 1024);
          ptx::mma_bf16(acc, adesc, ptx::smem_desc_sw128(simg + kk * 2048, 8192, 1024), IDESC_N2,
                        kk ? 1u : 0u);
          ptx::mma_bf16(acc, adesc, ptx::smem_desc_sw128(simg + 8192 + kk * 2048, 8192, 1024),
                        IDESC_N2, 1u);
        }
        if (!wait_bounded(pm_bar, cph, flag, kFlagApplyTimeout, &s_abort)) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16_ta(acc, tmem + TPM + 8u * kk,
                           ptx::smem_desc_sw128(vt + kk * 2048, HALF, 1024), IDESC_N3, 1u);
        ptx::mma_commit(numfull_bar(b));
        ptx::mma_commit(empty_bar(it.stage));
      }
      ptx::mma_commit(done_bar);
      wait_bounded(done_bar, 0, flag, kFlagApplyTimeout, &s_abort);
    }
  } else {
    // ---------------- math warps ----------------
    const int tt = threadIdx.x - 64;
    const int mw = warp - 2;
    // transform layout: chunk column cc (8 dims), rows 64 rh + lane and + 32
    const int cc = mw & 7, rh = mw >> 3;
    // tensor-memory layout: lane quadrant q4 (rows 32 q4 ..), 4 warps per quadrant
    const int q4 = warp & 3, jw = (warp - 2) >> 2;
    const uint32_t lane_bits = (uint32_t)(32 * q4) << 16;
    const uint32_t tmem = *s_tmem;
    if (ROPE) {
      for (int e = tt; e < rope.entries; e += kMath) s_tab[e] = gtab[e];
    }
    ChunkCol col{};
    if (ROPE) col = chunk_col(rope, cc);

    // ---- start state: the earlier CTAs' partials of the first head ----
    TileIter it;
    it.init(u0, sc.tps, stages);
    {
      const int seg0 = it.seg;
      const int first = cta_of_unit(sc, (long long)seg0 * sc.tps);
      const int np = it.tile == 0 ? 0 : cta - first;   // a CTA that starts a head starts at zero
      const float* pbase = partials + (long long)seg0 * sc.maxc * DD1;
      // S rows a = 16 q4 + lane (lanes 0-15), columns d = 16 jw .. 16 jw + 15
      const int a = 16 * q4 + (lane & 15);
      // S[a][d] = column d of S, row a (at d * D + a of a partial): the 16
      // loads of a partial in flight together, the partials added in order
      float acc[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] = 0.f;
      float zacc = 0.f;
      for (int k = 0; k < np; ++k) {
        const float* pk = pbase + (long long)k * DD1 + a;
        float t[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) t[e] = __ldcg(pk + (16 * jw + e) * D);
        const float tz = jw == 0 ? __ldcg(pk + D * D) : 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] += t[e];
        zacc += tz;
      }
      uint32_t sv[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) sv[e] = __float_as_uint(acc[e]);
      if (lane < 16) {
        uint8_t* img = sm + P.off_simg + 16384u;   // image of the start state: buffer 1
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4 hi, lo;
          split_hilo8(sv + 8 * h, hi, lo);
          *reinterpret_cast<uint4*>(img + simg_chunk(a, 2 * jw + h)) = hi;
          *reinterpret_cast<uint4*>(img + 8192 + simg_chunk(a, 2 * jw + h)) = lo;
        }
        if (jw == 0) s_zs[a] = zacc;
      }
      tmem_st_32x32_x16(tmem + lane_bits + TS + 16u * jw, sv);
      // the blocks of P_m above the diagonal block row stay zero
      if (jw > q4) {
        uint32_t zero[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) zero[e] = 0u;
        tmem_st_32x32_x16(tmem + lane_bits + TPM + 16u * jw, zero);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::fence_proxy_async();
      ptx::bar_sync(1, kMath);   // table, start image and z complete
      ptx::mbar_arrive(simg_bar);   // phase 0: the state before the first chunk
    }
    float zr[8];   // running key sum of this thread's chunk column (dims 8 cc ..)
#pragma unroll
    for (int e = 0; e < 8; ++e) zr[e] = s_zs[8 * cc + e];

    int pend = -1, pend_seg = 0, pend_tile = 0;
    uint4 gv[2];
    gv[0] = gv[1] = make_uint4(0u, 0u, 0u, 0u);
    // out rows of chunk pc: num / den (* sigmoid(g)), rounded to bf16
    auto epilogue = [&](int pc, int pseg, int ptile) {
      const int eb = pc & 1;
      const bool rdy = wait_bounded(numfull_bar(eb), (uint32_t)((pc >> 1) & 1), flag,
                                    kFlagApplyTimeout, &s_abort);
      ptx::tc_fence_after();
      uint32_t vh[16];
      tmem_ld_cols<16>(tmem + lane_bits + TNUM + (uint32_t)eb * 64u + 16u * jw, vh);
      ptx::tmem_wait_ld();
      const int row = 32 * q4 + lane;
      const int r = ptile * TM + row;
      if (rdy && r < L) {
        // the 8 chunk columns' parts of this row's denominator (column-major:
        // consecutive rows in consecutive banks)
        const float* dp = s_den + (pc % 3) * 8 * TM + row;
        float dv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) dv[e] = dp[e * TM];
        const float den = eps + (((dv[0] + dv[1]) + (dv[2] + dv[3])) + ((dv[4] + dv[5]) + (dv[6] + dv[7])));
        const float inv = 1.f / den;
        const uint64_t inv2 = ptx::f2(inv, inv);
        uint4* dst = reinterpret_cast<uint4*>(out + scd.out_row(pseg, L, r, D) + 16 * jw);
#pragma unroll
        for (int k4 = 0; k4 < 2; ++k4) {
          float o[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint64_t hv = ptx::f2(__uint_as_float(vh[8 * k4 + 2 * e]),
                                        __uint_as_float(vh[8 * k4 + 2 * e + 1]));
            ptx::f2_split(ptx::mul2(hv, inv2), o[2 * e], o[2 * e + 1]);
          }
          if (GATE) {
            const uint32_t gw[4] = {gv[k4].x, gv[k4].y, gv[k4].z, gv[k4].w};
            constexpr float kNegLog2e = -1.4426950408889634f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              o[2 * e] *= ptx::rcp_approx(1.f + ptx::ex2_approx(kNegLog2e * ptx::bf16_lo(gw[e])));
              o[2 * e + 1] *=
                  ptx::rcp_approx(1.f + ptx::ex2_approx(kNegLog2e * ptx::bf16_hi(gw[e])));
            }
          }
          dst[k4] = make_uint4(ptx::pack_bf16x2(o[0], o[1]), ptx::pack_bf16x2(o[2], o[3]),
                               ptx::pack_bf16x2(o[4], o[5]), ptx::pack_bf16x2(o[6], o[7]));
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(numfree_bar(eb));
    };
    auto load_gate = [&](int pseg, int ptile) {
      const int r = ptile * TM + 32 * q4 + lane;
      if (GATE && r < L) {
        const uint4* src = reinterpret_cast<const uint4*>(g + scd.out_row(pseg, L, r, D) + 16 * jw);
        gv[0] = __ldg(src);
        gv[1] = __ldg(src + 1);
      }
    };
    // ---- A(ca): RoPE(phi q), RoPE(phi k) in place for chunk ca (the TMA
    // stage of itA); running key sums and the chunk's denominators ----
    TileIter itA = it;
    auto transform = [&](long long ca) {
      const int stage = itA.stage;
      const uint32_t qt = base + stage * 3u * kCTile, kt = qt + kCTile;
      if (itA.tile == 0) {   // a head starts: no earlier keys
#pragma unroll
        for (int e = 0; e < 8; ++e) zr[e] = 0.f;
      }
      const bool ok = wait_bounded(full_bar(stage), itA.phase, flag, kFlagApplyTimeout, &s_abort);
      (void)ok;
      float pq[2][8], pk[2][8];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = 64 * rh + 32 * i + lane;
        const uint32_t off = r * 128 + ((cc ^ (r & 7)) << 4);
        const float4* cs = ROPE ? reinterpret_cast<const float4*>(
                                      s_tab + s_pos[(stage * 3 + col.ax) * TM + r] + col.pair_off)
                                : nullptr;
        uint64_t xy[4];
        uint32_t m[4];
        const uint4 oq = phi_rope<ROPE>(ptx::ld_shared_v4(qt + off), cs, xy, m);
        ptx::st_shared_v4(qt + off, oq);
        // xy = {(d0, d2), (d4, d6), (d1, d3), (d5, d7)} of the chunk's 8 dims
        ptx::f2_split(xy[0], pq[i][0], pq[i][2]);
        ptx::f2_split(xy[1], pq[i][4], pq[i][6]);
        ptx::f2_split(xy[2], pq[i][1], pq[i][3]);
        ptx::f2_split(xy[3], pq[i][5], pq[i][7]);
        const uint4 ok4 = phi_rope<ROPE>(ptx::ld_shared_v4(kt + off), cs, xy, m);
        ptx::st_shared_v4(kt + off, ok4);
        ptx::f2_split(xy[0], pk[i][0], pk[i][2]);
        ptx::f2_split(xy[1], pk[i][4], pk[i][6]);
        ptx::f2_split(xy[2], pk[i][1], pk[i][3]);
        ptx::f2_split(xy[3], pk[i][5], pk[i][7]);
      }
      ptx::fence_proxy_async();
      ptx::mbar_arrive(kready_bar(stage));
      // inclusive key sums down this warp's 64 rows, then across the two halves
      const int wb = (int)(ca & 1);
      warp_scan8(pk[0], lane);
      warp_scan8(pk[1], lane);
      float* wt = s_wtot + ((wb * 2 + rh) * 8 + cc) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        pk[1][e] += __shfl_sync(0xffffffffu, pk[0][e], 31);
        if (lane == 31) wt[e] = pk[1][e];
      }
      ptx::bar_sync(2, kMath);
      const float* w0 = s_wtot + ((wb * 2 + 0) * 8 + cc) * 8;
      const float* w1 = s_wtot + ((wb * 2 + 1) * 8 + cc) * 8;
      float dq[2] = {0.f, 0.f};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float base_e = zr[e] + (rh ? w0[e] : 0.f);
        dq[0] = fmaf(pq[0][e], base_e + pk[0][e], dq[0]);
        dq[1] = fmaf(pq[1][e], base_e + pk[1][e], dq[1]);
        zr[e] += w0[e] + w1[e];
      }
      const int db = (int)(ca % 3);
#pragma unroll
      for (int i = 0; i < 2; ++i) s_den[(db * 8 + cc) * TM + 64 * rh + 32 * i + lane] = dq[i];
      itA.next();
    };

    const long long nch = u1 - u0;
    transform(0);
    for (long long c = 0; c < nch; ++c) {
      const int b = (int)(c & 1);
      const uint32_t cph = (uint32_t)(c & 1);
      const int seg = it.seg, tile = it.tile;
      // the next chunk's transform while the tensor cores finish this one
      if (c + 1 < nch) transform(c + 1);
      // ---- B: the previous chunk's epilogue ----
      if (pend >= 0) {
        load_gate(pend_seg, pend_tile);
        epilogue(pend, pend_seg, pend_tile);
      }
      // ---- C: P masked to j <= i, as the bf16 A operand of P_m V ----
      {
        const bool rdy = wait_bounded(pfull_bar, cph, flag, kFlagApplyTimeout, &s_abort);
        ptx::tc_fence_after();
        if (jw <= q4) {
          uint32_t pv[32], pk2[16];
          tmem_ld_cols<32>(tmem + lane_bits + TP + 32u * jw, pv);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float p0 = __uint_as_float(pv[2 * e]), p1 = __uint_as_float(pv[2 * e + 1]);
            if (jw == q4) {   // the diagonal block: column 32 jw + k is kept for k <= lane
              if (2 * e > lane) p0 = 0.f;
              if (2 * e + 1 > lane) p1 = 0.f;
            }
            pk2[e] = ptx::pack_bf16x2(p0, p1);
          }
          tmem_st_32x32_x16(tmem + lane_bits + TPM + 16u * jw, pk2);
          ptx::tmem_wait_st();
        }
        (void)rdy;
        ptx::tc_fence_before();
        ptx::mbar_arrive(pm_bar);
      }
      // ---- D: image of the state after this chunk (or the zero state when the
      // next chunk starts a new head) for the next chunk's A S ----
      {
        const bool rdy = wait_bounded(sfull_bar, cph, flag, kFlagApplyTimeout, &s_abort);
        ptx::tc_fence_after();
        (void)rdy;
        const bool restart = tile + 1 == sc.tps;   // the next chunk (if any) starts a head
        uint32_t sv[16];
        tmem_ld_cols<16>(tmem + lane_bits + TS + 16u * jw, sv);
        ptx::tmem_wait_ld();
        if (restart) {
#pragma unroll
          for (int e = 0; e < 16; ++e) sv[e] = 0u;
          tmem_st_32x32_x16(tmem + lane_bits + TS + 16u * jw, sv);
          ptx::tmem_wait_st();
        }
        if (lane < 16) {
          const int a = 16 * q4 + lane;
          uint8_t* img = sm + P.off_simg + (uint32_t)b * 16384u;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint4 hi, lo;
            split_hilo8(sv + 8 * h, hi, lo);
            *reinterpret_cast<uint4*>(img + simg_chunk(a, 2 * jw + h)) = hi;
            *reinterpret_cast<uint4*>(img + 8192 + simg_chunk(a, 2 * jw + h)) = lo;
          }
        }
        ptx::tc_fence_before();
        ptx::fence_proxy_async();
        ptx::mbar_arrive(simg_bar);
      }
      pend = (int)c;
      pend_seg = seg;
      pend_tile = tile;
      it.next();
    }
    if (pend >= 0) {
      load_gate(pend_seg, pend_tile);
      epilogue(pend, pend_seg, pend_tile);
    }
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(*s_tmem, TMEM_COLS);
  }
}

}  // namespace la

namespace la {

// Token-causal forward on the tensor cores (D = 64): the state build writes
// one partial per (head, CTA) and no image; causal_tc reads them.
inline la_status causal_run(const TcArgs& a) {
  const int entries = a.rope.on ? a.rope.entries : 0;
  const Sched& sc = a.sc;
  SegCoords scd;
  scd.bnhd = a.bnhd;
  scd.H = a.H > 0 ? a.H : 1;
  scd.nblk = sc.nblk;
  scd.div_nblk = make_fastdiv(sc.nblk);
  scd.div_h = make_fastdiv(scd.H);
  CUtensorMap mk, mv, mq;
  if (!make_map(&mk, a.k, 64, sc.L, sc.nseg, tc_state_tile_c(64), scd) ||
      !make_map(&mv, a.v, 64, sc.L, sc.nseg, tc_state_tile_c(64), scd) ||
      !make_map(&mq, a.q, 64, sc.L, sc.nseg, tc_state_tile_c(64), scd))
    return LA_ERR_CUDA;
  la_status st;
  const int s1 = pick_state_stages(64, entries);
  const StatePlan p1 = state_plan(64, entries, s1);
  auto k1 = a.rope.on ? state_build_tc<64, true> : state_build_tc<64, false>;
  if ((st = tc_smem_attr(k1, p1.total)) != LA_OK) return st;
  if ((st = tc_mark(a, 0)) != LA_OK) return st;
  st = launch_pdl(k1, dim3(sc.G), dim3(kTcThreadsState), p1.total, a.stream, mk, mv, a.rope, sc,
                  scd, s1, a.part, a.gtab, a.flag, static_cast<int*>(nullptr),
                  static_cast<uint8_t*>(nullptr), static_cast<float*>(nullptr),
                  static_cast<float*>(nullptr), 0, 0);
  if (st != LA_OK) return st;
  if ((st = tc_mark(a, 1)) != LA_OK) return st;
  if ((st = tc_mark(a, 2)) != LA_OK) return st;
  const int s2 = pick_causal_stages(entries);
  if (s2 == 0) return LA_ERR_UNSUPPORTED;
  const CausalPlan p2 = causal_plan(entries, s2);
  const bool gate = a.g != nullptr;
  auto k2 = a.rope.on ? (gate ? causal_tc<true, true> : causal_tc<true, false>)
                      : (gate ? causal_tc<false, true> : causal_tc<false, false>);
  if ((st = tc_smem_attr(k2, p2.total)) != LA_OK) return st;
  st = launch_pdl(k2, dim3(sc.G), dim3(kCausalTcThreads), p2.total, a.stream, mq, mk, mv, a.rope,
                  sc, scd, s2, static_cast<const float*>(a.part),
                  static_cast<const float2*>(a.gtab), static_cast<const __nv_bfloat16*>(a.g),
                  static_cast<__nv_bfloat16*>(a.out), a.eps, a.flag);
  if (st != LA_OK) return st;
  return tc_mark(a, 3);
}

// Whether a token-causal call takes the tensor-core kernels: bf16, D = 64,
// RoPE widths in multiples of 8, and the kernels' shared memory within budget.
inline bool causal_tc_supported(bool bf16, int D, int rope, int dt, int dh, int dw, int entries) {
  if (!bf16 || D != 64) return false;
  if (rope && ((dt % 8) || (dh % 8) || (dw % 8))) return false;
  const int e = rope ? entries : 0;
  return pick_state_stages(64, e) > 0 && pick_causal_stages(e) > 0;
}

}  // namespace la

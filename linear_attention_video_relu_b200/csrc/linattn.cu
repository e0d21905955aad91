// linattn.cu -- host side of the C ABI declared in include/linattn.h:
// argument checks, the work plan, the workspace carve-up and the launches.
//
// A forward follows the factorised form of Eq. 2 and the block recursion of
// Eq. 3 / Algorithm 1 (SANA-Video paper-graph page, section 3.4) in up to
// three launches on the caller's stream:
//   1. state build  (per contiguous tile range: partial S, z of every segment
//                    the range touches; also the RoPE cos/sin table)
//   2. reduce       (fixed-order sum of the partials per segment, then the
//                    block-causal running sum, or the carried state) -- on
//                    the tensor-core path folded into the state build when
//                    every head is one segment
//   3. apply        (out = RoPE(phi q) S / (phi q . z + eps), gate)
// The token-causal mode runs on the tensor cores at bf16 and D = 64 (the state
// build's partials, then causal_tc carrying the running state through each
// CTA's range), else on the CUDA-core kernels with 32-token chunks as
// segments and a chunked apply step.
#include "linattn.h"

#include <limits.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "causal.cuh"
#include "common.cuh"
#include "simt.cuh"
#include "tc.cuh"

using namespace la;

namespace {

constexpr size_t kAlign = 256;
// Control block at the start of every workspace: the bounded-wait flag word,
// then one arrival counter per segment (at most kMaxCounters of them).
constexpr size_t kCounterOffset = 256;
constexpr int kMaxCounters = (int)((LA_WORKSPACE_CONTROL_BYTES - kCounterOffset) / sizeof(int));

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Plan {
  bool tc;             // tensor-core kernels
  bool causal;         // token-causal mode (CUDA-core kernels, chunked)
  Rope rope;
  Sched sc;
  long long heads;
  long long nq;        // query tokens per head (N; the query length of a cross-attention)
  int lq;              // query rows per segment (sc.L, or nq for a cross-attention)
  int apply_tps;       // SIMT apply: tiles per segment
  int sms;             // SM count of the device
  Layout lay;          // memory order of q, k, v, gate, out
  size_t off_flag, off_tab, off_part, off_apply, total;
};

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
  return a0 < b0 + nb && b0 < a0 + na;
}

la_status device_sms(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return LA_ERR_CUDA; }
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  return LA_OK;
}

// Checks that need no device. `one_block`: lin_attn_block_step semantics.
la_status check_params(const la_params* p, bool one_block) {
  if (!p) return LA_ERR_INVALID_ARG;
  if (p->B < 0 || p->H < 0 || p->N < 0) return LA_ERR_INVALID_ARG;
  if (p->D != 32 && p->D != 64 && p->D != 112 && p->D != 128) return LA_ERR_INVALID_ARG;
  if (p->dtype != LA_F32 && p->dtype != LA_BF16) return LA_ERR_INVALID_ARG;
  if (p->layout != LA_LAYOUT_BHND && p->layout != LA_LAYOUT_BNHD) return LA_ERR_INVALID_ARG;
  if (!one_block) {
    if (p->mode != LA_BIDIRECTIONAL && p->mode != LA_BLOCK_CAUSAL && p->mode != LA_TOKEN_CAUSAL)
      return LA_ERR_INVALID_ARG;
    if (p->mode == LA_BLOCK_CAUSAL &&
        (p->block_tokens < 1 || (p->N > 0 && p->N % p->block_tokens != 0)))
      return LA_ERR_INVALID_ARG;
  }
  if (!(p->eps >= 0.f) || isinf(p->eps)) return LA_ERR_INVALID_ARG;
  if (p->rope) {
    if (p->rope_dt < 0 || p->rope_dh < 0 || p->rope_dw < 0) return LA_ERR_INVALID_ARG;
    if ((p->rope_dt | p->rope_dh | p->rope_dw) & 1) return LA_ERR_INVALID_ARG;
    if (p->rope_dt + p->rope_dh + p->rope_dw != p->D) return LA_ERR_INVALID_ARG;
    if (p->grid_t < 1 || p->grid_h < 1 || p->grid_w < 1) return LA_ERR_INVALID_ARG;
    if ((long long)p->grid_t * p->grid_h * p->grid_w != (long long)p->N) return LA_ERR_INVALID_ARG;
    if (!(p->rope_theta > 0.0) || isinf(p->rope_theta)) return LA_ERR_INVALID_ARG;
    long long entries = (long long)p->grid_t * rope_stride(p->rope_dt / 2) +
                        (long long)p->grid_h * rope_stride(p->rope_dh / 2) +
                        (long long)p->grid_w * rope_stride(p->rope_dw / 2);
    if (entries > kMaxRopeEntries) return LA_ERR_UNSUPPORTED;
  }
  long long heads = (long long)p->B * p->H;
  if (heads > (1LL << 24)) return LA_ERR_UNSUPPORTED;
  // segments (head x block, or head x token chunk) are indexed with int
  long long nblk = 1;
  if (!one_block && p->mode == LA_BLOCK_CAUSAL && p->N > 0) nblk = p->N / p->block_tokens;
  if (!one_block && p->mode == LA_TOKEN_CAUSAL) nblk = (p->N + kCausalChunk - 1) / kCausalChunk;
  if (heads * nblk > (long long)INT_MAX) return LA_ERR_UNSUPPORTED;
  return LA_OK;
}

bool want_tc(const la_params* p, bool one_block) {
  // 112-wide heads run padded on the 128 kernels, whose carried-state I/O is
  // 128 wide: block steps at D = 112 stay on the CUDA-core kernels
  if (one_block && p->D == 112) return false;
  const int entries = p->rope ? p->grid_t * rope_stride(p->rope_dt / 2) +
                                    p->grid_h * rope_stride(p->rope_dh / 2) +
                                    p->grid_w * rope_stride(p->rope_dw / 2)
                              : 0;
  if (!one_block && p->mode == LA_TOKEN_CAUSAL)   // tensor cores at D = 64 only
    return causal_tc_supported(p->dtype == LA_BF16, p->D, p->rope, p->rope_dt, p->rope_dh,
                               p->rope_dw, entries);
  return tc_supported(p->dtype == LA_BF16, p->D, p->rope, p->rope_dt, p->rope_dh, p->rope_dw,
                      entries);
}

// Plan for a call of p (one_block: the N tokens are a single block of a
// block step). Needs the device only for its SM count.
la_status make_plan(const la_params* p, bool one_block, int t_offset, Plan* pl) {
  la_status st = check_params(p, one_block);
  if (st != LA_OK) return st;
  int sms = 0;
  st = device_sms(&sms);
  if (st != LA_OK) return st;
  memset(pl, 0, sizeof(*pl));
  pl->tc = want_tc(p, one_block);
  pl->sms = sms;
  pl->heads = (long long)p->B * p->H;
  pl->lay.bnhd = p->layout == LA_LAYOUT_BNHD ? 1 : 0;
  pl->lay.H = p->H > 0 ? p->H : 1;
  pl->lay.div_h = make_fastdiv(pl->lay.H);

  Rope& r = pl->rope;
  r.on = p->rope ? 1 : 0;
  if (r.on) {
    r.T = p->grid_t;
    r.Hg = p->grid_h;
    r.Wg = p->grid_w;
    r.t_offset = t_offset;
    r.half[0] = p->rope_dt / 2;
    r.half[1] = p->rope_dh / 2;
    r.half[2] = p->rope_dw / 2;
    r.pair_base[0] = 0;
    r.pair_base[1] = r.half[0];
    r.pair_base[2] = r.half[0] + r.half[1];
    for (int a = 0; a < 3; ++a) r.stride[a] = rope_stride(r.half[a]);
    r.tab_off[0] = 0;
    r.tab_off[1] = r.T * r.stride[0];
    r.tab_off[2] = r.tab_off[1] + r.Hg * r.stride[1];
    r.entries = r.tab_off[2] + r.Wg * r.stride[2];
    r.theta = p->rope_theta;
    r.div_hw = make_fastdiv(r.Hg * r.Wg);
    r.div_w = make_fastdiv(r.Wg);
    // constants of the rotary parameterisation: theta^(-2m/d) / pi per pair,
    // split into float hi + lo
    for (int a = 0; a < 3; ++a) {
      for (int m = 0; m < r.half[a]; ++m) {
        const double v = pow(r.theta, -(double)m / (double)r.half[a]) / M_PI;
        r.inv_pi_hi[r.pair_base[a] + m] = (float)v;
        r.inv_pi_lo[r.pair_base[a] + m] = (float)(v - (double)(float)v);
      }
    }
  }

  Sched& sc = pl->sc;
  const int N = p->N;
  // token-causal: on the CUDA-core kernels, segments of kCausalChunk tokens
  // (the last one ragged); on the tensor cores, one segment per head (the
  // apply kernel carries the running state through each CTA's range)
  pl->causal = !one_block && p->mode == LA_TOKEN_CAUSAL;
  sc.L = (pl->causal && !pl->tc)
             ? kCausalChunk
             : ((!one_block && p->mode == LA_BLOCK_CAUSAL) ? p->block_tokens : N);
  if (sc.L < 1) sc.L = 1;
  sc.nblk = (N + sc.L - 1) / sc.L;
  if (sc.nblk < 1) sc.nblk = 1;
  sc.nseg = (int)(pl->heads * sc.nblk);
  const int Dk = pl->tc ? tc_kernel_dim(p->D) : p->D;   // head dim the kernels run at
  sc.TT = pl->tc ? tc_state_tile(Dk) : kSimtTileState;
  sc.tps = (sc.L + sc.TT - 1) / sc.TT;
  sc.U = (long long)sc.nseg * sc.tps;
  long long G = pl->tc ? (long long)sms * tc_state_ctas_per_sm(p->D) : 2LL * sms;
  if (G > sc.U) G = sc.U;
  if (G < 1) G = 1;
  sc.G = (int)G;
  sc.fastU = sc.U > 0 && sc.U * sc.G < (1LL << 31);
  sc.divU = make_fastdiv(sc.fastU ? (int)sc.U : 1);
  sc.maxc = 1;
  if (sc.U > 0) {
    for (int s = 0; s < sc.nseg; ++s) {
      long long ub = (long long)s * sc.tps;
      int c = cta_of_unit(sc, ub + sc.tps - 1) - cta_of_unit(sc, ub) + 1;
      if (c > sc.maxc) sc.maxc = c;
    }
  }
  pl->nq = N;
  pl->lq = sc.L;
  pl->apply_tps = (sc.L + kSimtTileApply - 1) / kSimtTileApply;

  const size_t dd1 = (size_t)Dk * (Dk + 1);
  size_t off = 0;
  pl->off_flag = off;                     // control block: flag word, then counters
  off += LA_WORKSPACE_CONTROL_BYTES;
  pl->off_tab = off;
  off += round_up((size_t)(r.on ? r.entries : 0) * sizeof(float2), kAlign);
  pl->off_part = off;
  off += round_up((size_t)sc.nseg * sc.maxc * dd1 * sizeof(float), kAlign);
  pl->off_apply = off;   // fp32 apply states (SIMT) or B-operand images (tensor cores)
  const size_t per_seg = pl->tc ? (size_t)image_bytes(Dk) : dd1 * sizeof(float);
  off += round_up((size_t)sc.nseg * per_seg, kAlign);
  pl->total = off;
  return LA_OK;
}

la_status check_tensor(const void* ptr, bool needed) {
  if (!needed) return LA_OK;
  if (!ptr) return LA_ERR_INVALID_ARG;
  if (!aligned16(ptr)) return LA_ERR_INVALID_ARG;
  return LA_OK;
}

la_status last_error() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

template <typename KernelT>
la_status set_smem(KernelT kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return LA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_UNSUPPORTED;
  }
  return LA_OK;
}

struct Launch {
  const la_params* p;
  const Plan* pl;
  const void *q, *k, *v, *g;
  void* out;
  unsigned char* ws;
  float* stS;
  float* stz;
  int use_state, commit, do_apply;
  cudaStream_t stream;
  void* const* events;   // optional: 4 events recorded around the launches
};

la_status mark(const Launch& L, int i) {
  if (!L.events || !L.events[i]) return LA_OK;
  if (cudaEventRecord(static_cast<cudaEvent_t>(L.events[i]), L.stream) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  return LA_OK;
}

template <int D, typename T>
la_status run_simt(const Launch& L) {
  const Plan& pl = *L.pl;
  float2* gtab = reinterpret_cast<float2*>(L.ws + pl.off_tab);
  float* part = reinterpret_cast<float*>(L.ws + pl.off_part);
  float* apply = reinterpret_cast<float*>(L.ws + pl.off_apply);
  const long long N = L.p->N;
  const int TT = kSimtTileState;
  size_t smem1 = 3 * (size_t)TT * D * sizeof(float) +
                 (size_t)(pl.rope.on ? pl.rope.entries : 0) * sizeof(float2);
  la_status st = set_smem(state_partial_simt<D, T>, smem1);
  if (st != LA_OK) return st;
  if ((st = mark(L, 0)) != LA_OK) return st;
  state_partial_simt<D, T><<<pl.sc.G, kSimtThreads, smem1, L.stream>>>(
      static_cast<const T*>(L.k), static_cast<const T*>(L.v), N, pl.lay, pl.rope, pl.sc, part,
      gtab);
  if ((st = last_error()) != LA_OK) return st;
  if ((st = mark(L, 1)) != LA_OK) return st;
  dim3 g2((D * (D + 1) + 255) / 256, (unsigned)(pl.heads < 65535 ? pl.heads : 65535));
  reduce_states<D><<<g2, 256, 0, L.stream>>>(part, pl.sc, apply, L.stS, L.stz, L.use_state,
                                              L.commit);
  if ((st = last_error()) != LA_OK) return st;
  if ((st = mark(L, 2)) != LA_OK) return st;
  if (!L.do_apply) return LA_OK;
  if (pl.causal) {
    const int C = kCausalChunk;
    size_t smemc = ((size_t)D * (D + 1) + 3 * (size_t)C * D + 2 * (size_t)C * (D + 1) +
                    2 * (size_t)C * C + C) * sizeof(float);
    if ((st = set_smem(apply_causal_simt<D, T>, smemc)) != LA_OK) return st;
    const int gc = pl.sc.nseg < (1 << 20) ? pl.sc.nseg : (1 << 20);
    apply_causal_simt<D, T><<<gc, kSimtThreads, smemc, L.stream>>>(
        static_cast<const T*>(L.q), static_cast<const T*>(L.k), static_cast<const T*>(L.v),
        static_cast<const T*>(L.g), static_cast<T*>(L.out), N, pl.lay, pl.rope, pl.sc.nblk,
        pl.sc.nseg, apply, gtab, L.p->eps);
    if ((st = last_error()) != LA_OK) return st;
    return mark(L, 3);
  }
  const int TA = kSimtTileApply;
  size_t smem3 = ((size_t)D * (D + 1) + 2 * (size_t)TA * D + TA) * sizeof(float);
  st = set_smem(apply_simt<D, T>, smem3);
  if (st != LA_OK) return st;
  dim3 g3(pl.apply_tps, pl.sc.nseg < 65535 ? pl.sc.nseg : 65535);
  apply_simt<D, T><<<g3, kSimtThreads, smem3, L.stream>>>(
      static_cast<const T*>(L.q), static_cast<const T*>(L.g), static_cast<T*>(L.out), pl.nq,
      pl.lay, pl.rope, pl.lq, pl.sc.nblk, pl.apply_tps, pl.sc.nseg, apply, gtab, L.p->eps);
  if ((st = last_error()) != LA_OK) return st;
  return mark(L, 3);
}

template <typename T>
la_status dispatch_simt(const Launch& L) {
  switch (L.p->D) {
    case 32: return run_simt<32, T>(L);
    case 64: return run_simt<64, T>(L);
    case 112: return run_simt<112, T>(L);
    case 128: return run_simt<128, T>(L);
  }
  return LA_ERR_UNSUPPORTED;
}

la_status run(const Launch& L) {
  if (L.pl->tc) {
    TcArgs a;
    a.D = L.p->D;
    a.N = L.p->N;
    a.Lq = L.pl->lq;
    a.rope = L.pl->rope;
    a.sc = L.pl->sc;
    a.heads = L.pl->heads;
    a.q = L.q;
    a.k = L.k;
    a.v = L.v;
    a.g = L.g;
    a.out = L.out;
    a.flag = reinterpret_cast<int*>(L.ws + L.pl->off_flag);
    a.counters = reinterpret_cast<int*>(L.ws + L.pl->off_flag + kCounterOffset);
    a.bnhd = L.pl->lay.bnhd;
    a.H = L.pl->lay.H;
    a.fused = L.pl->sc.nblk == 1 && L.pl->sc.nseg <= kMaxCounters;
    a.gtab = reinterpret_cast<float2*>(L.ws + L.pl->off_tab);
    a.part = reinterpret_cast<float*>(L.ws + L.pl->off_part);
    a.apply = reinterpret_cast<float*>(L.ws + L.pl->off_apply);
    a.stS = L.stS;
    a.stz = L.stz;
    a.use_state = L.use_state;
    a.commit = L.commit;
    a.do_apply = L.do_apply;
    a.eps = L.p->eps;
    a.stream = L.stream;
    a.events = L.events;
    if (L.pl->causal) return causal_run(a);
    return tc_run(a, L.pl->sms);
  }
  if (L.p->dtype == LA_BF16) return dispatch_simt<__nv_bfloat16>(L);
  return dispatch_simt<float>(L);
}

size_t elt_size(const la_params* p) { return p->dtype == LA_BF16 ? 2 : 4; }

la_status check_io(const la_params* p, const void* q, const void* k, const void* v,
                   const void* g, const void* out, bool need_q) {
  la_status st;
  if ((st = check_tensor(k, true)) != LA_OK) return st;
  if ((st = check_tensor(v, true)) != LA_OK) return st;
  if ((st = check_tensor(q, need_q)) != LA_OK) return st;
  if ((st = check_tensor(out, need_q)) != LA_OK) return st;
  if (g && !aligned16(g)) return LA_ERR_INVALID_ARG;
  if (need_q) {
    size_t bytes = (size_t)p->B * p->H * p->N * p->D * elt_size(p);
    if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) ||
        overlaps(out, bytes, v, bytes) || overlaps(out, bytes, g, bytes))
      return LA_ERR_INVALID_ARG;
  }
  return LA_OK;
}

la_status check_workspace(const Plan& pl, const void* ws, size_t bytes) {
  if (!ws || ((uintptr_t)ws % kAlign) != 0) return LA_ERR_WORKSPACE;
  if (bytes < pl.total) return LA_ERR_WORKSPACE;
  return LA_OK;
}

la_status check_state(const la_params* p, const la_state* st) {
  if (!st || !st->S || !st->z) return LA_ERR_INVALID_ARG;
  if (!aligned16(st->S) || !aligned16(st->z)) return LA_ERR_INVALID_ARG;
  if (st->B != p->B || st->H != p->H || st->D != p->D) return LA_ERR_INVALID_ARG;
  return LA_OK;
}

la_status block_common(const la_params* p, la_state* st, int t_offset, const void* q,
                       const void* k, const void* v, const void* gate, void* out, int commit,
                       void* workspace, size_t workspace_bytes, void* stream, bool do_apply) {
  la_status s = check_params(p, true);
  if (s != LA_OK) return s;
  if ((s = check_state(p, st)) != LA_OK) return s;
  if (t_offset < 0) return LA_ERR_INVALID_ARG;
  if ((long long)p->B * p->H * p->N == 0) return LA_OK;
  if ((s = check_io(p, q, k, v, gate, out, do_apply)) != LA_OK) return s;
  // The state is read and (commit) updated in place while q, k, v and gate
  // are still being read and out written: none of them may share its bytes,
  // and S and z may not share bytes with each other.
  const size_t sbytes = (size_t)p->B * p->H * p->D * p->D * sizeof(float);
  const size_t zbytes = (size_t)p->B * p->H * p->D * sizeof(float);
  const size_t tbytes = (size_t)p->B * p->H * p->N * p->D * elt_size(p);
  if (overlaps(st->S, sbytes, st->z, zbytes)) return LA_ERR_INVALID_ARG;
  const void* io[5] = {q, k, v, gate, out};
  for (const void* t : io)
    if (overlaps(t, tbytes, st->S, sbytes) || overlaps(t, tbytes, st->z, zbytes))
      return LA_ERR_INVALID_ARG;
  Plan pl;
  if ((s = make_plan(p, true, t_offset, &pl)) != LA_OK) return s;
  if ((s = check_workspace(pl, workspace, workspace_bytes)) != LA_OK) return s;
  Launch L{p, &pl, q, k, v, gate, out, static_cast<unsigned char*>(workspace), st->S, st->z,
           1, commit ? 1 : 0, do_apply ? 1 : 0, static_cast<cudaStream_t>(stream), nullptr};
  return run(L);
}

// Plan of a linear cross-attention: the state is built from the n_kv keys and
// values of each head (one segment per head), and applied to the p->N queries.
la_status cross_plan(const la_params* p, int n_kv, Plan* pl) {
  la_status s = check_params(p, false);
  if (s != LA_OK) return s;
  if (p->rope || p->mode != LA_BIDIRECTIONAL || n_kv < 1) return LA_ERR_INVALID_ARG;
  la_params pk = *p;
  pk.N = n_kv;
  if ((s = make_plan(&pk, false, 0, pl)) != LA_OK) return s;
  pl->nq = p->N;
  pl->lq = p->N;
  pl->apply_tps = (p->N + kSimtTileApply - 1) / kSimtTileApply;
  return LA_OK;
}

// ---- fixed scratch for lin_attn_forward_noalloc ----------------------------
//
// The one device array behind lin_attn_forward_noalloc. In host code its name
// is only a stand-in for the symbol: the device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices];   // set once a lookup on that device succeeded

// Device address of the scratch array on the current device. Only a
// successful lookup is kept: a failed one (say, a call made before the
// context could be created) returns LA_ERR_CUDA and is tried again by the
// next call.
la_status noalloc_scratch(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return LA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return LA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return LA_OK;
}

}  // namespace

extern "C" {

la_status lin_attn_workspace_size(const la_params* p, size_t* bytes) {
  if (!bytes) return LA_ERR_INVALID_ARG;
  Plan pl;
  la_status s = make_plan(p, false, 0, &pl);
  if (s != LA_OK) return s;
  *bytes = pl.total;
  return LA_OK;
}

la_status lin_attn_block_step_workspace_size(const la_params* p, size_t* bytes) {
  if (!bytes) return LA_ERR_INVALID_ARG;
  Plan pl;
  la_status s = make_plan(p, true, 0, &pl);
  if (s != LA_OK) return s;
  *bytes = pl.total;
  return LA_OK;
}

la_status lin_attn_forward(const la_params* p, const void* q, const void* k, const void* v,
                           const void* gate, void* out, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return lin_attn_forward_timed(p, q, k, v, gate, out, workspace, workspace_bytes, stream,
                                nullptr);
}

la_status lin_attn_forward_timed(const la_params* p, const void* q, const void* k, const void* v,
                                 const void* gate, void* out, void* workspace,
                                 size_t workspace_bytes, void* stream, void* const* events) {
  la_status s = check_params(p, false);
  if (s != LA_OK) return s;
  if ((long long)p->B * p->H * p->N == 0) return LA_OK;
  if ((s = check_io(p, q, k, v, gate, out, true)) != LA_OK) return s;
  Plan pl;
  if ((s = make_plan(p, false, 0, &pl)) != LA_OK) return s;
  if ((s = check_workspace(pl, workspace, workspace_bytes)) != LA_OK) return s;
  Launch L{p, &pl, q, k, v, gate, out, static_cast<unsigned char*>(workspace), nullptr, nullptr,
           0, 0, 1, static_cast<cudaStream_t>(stream), events};
  return run(L);
}

la_status lin_attn_cross_workspace_size(const la_params* p, int n_kv, size_t* bytes) {
  if (!bytes) return LA_ERR_INVALID_ARG;
  Plan pl;
  la_status s = cross_plan(p, n_kv, &pl);
  if (s != LA_OK) return s;
  *bytes = pl.total;
  return LA_OK;
}

la_status lin_attn_cross_forward(const la_params* p, int n_kv, const void* q, const void* k,
                                 const void* v, const void* gate, void* out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  la_status s = check_params(p, false);
  if (s != LA_OK) return s;
  if (p->rope || p->mode != LA_BIDIRECTIONAL || n_kv < 1) return LA_ERR_INVALID_ARG;
  if ((long long)p->B * p->H * p->N == 0) return LA_OK;
  if ((s = check_tensor(q, true)) != LA_OK) return s;
  if ((s = check_tensor(k, true)) != LA_OK) return s;
  if ((s = check_tensor(v, true)) != LA_OK) return s;
  if ((s = check_tensor(out, true)) != LA_OK) return s;
  if (gate && !aligned16(gate)) return LA_ERR_INVALID_ARG;
  const size_t heads = (size_t)p->B * p->H;
  const size_t qb = heads * p->N * p->D * elt_size(p);
  const size_t kb = heads * (size_t)n_kv * p->D * elt_size(p);
  if (overlaps(out, qb, q, qb) || overlaps(out, qb, k, kb) || overlaps(out, qb, v, kb) ||
      overlaps(out, qb, gate, qb))
    return LA_ERR_INVALID_ARG;
  Plan pl;
  if ((s = cross_plan(p, n_kv, &pl)) != LA_OK) return s;
  if ((s = check_workspace(pl, workspace, workspace_bytes)) != LA_OK) return s;
  la_params pk = *p;
  pk.N = n_kv;
  Launch L{&pk, &pl, q, k, v, gate, out, static_cast<unsigned char*>(workspace), nullptr,
           nullptr, 0, 0, 1, static_cast<cudaStream_t>(stream), nullptr};
  return run(L);
}

la_status lin_attn_forward_noalloc(const la_params* p, const void* q, const void* k,
                                   const void* v, const void* gate, void* out, void* stream) {
  la_status s = check_params(p, false);
  if (s != LA_OK) return s;
  if ((long long)p->B * p->H * p->N == 0) return LA_OK;
  if ((s = check_io(p, q, k, v, gate, out, true)) != LA_OK) return s;
  Plan pl;
  if ((s = make_plan(p, false, 0, &pl)) != LA_OK) return s;
  if (pl.total > (size_t)LA_NOALLOC_SCRATCH_BYTES) return LA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != LA_OK) return s;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // the scratch starts zeroed; a call that gave up a bounded wait may leave
  // its control block dirty, and this path has no status query, so it is
  // cleared before every call
  if (cudaMemsetAsync(static_cast<unsigned char*>(scratch) + pl.off_flag, 0,
                      LA_WORKSPACE_CONTROL_BYTES, cs) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  Launch L{p, &pl, q, k, v, gate, out, static_cast<unsigned char*>(scratch), nullptr, nullptr,
           0, 0, 1, cs, nullptr};
  return run(L);
}

la_status lin_attn_state_init(la_state* st, int B, int H, int D, float* S, float* z) {
  if (!st || B < 0 || H < 0 || (D != 32 && D != 64 && D != 112 && D != 128))
    return LA_ERR_INVALID_ARG;
  if (!S || !z || !aligned16(S) || !aligned16(z)) return LA_ERR_INVALID_ARG;
  st->S = S;
  st->z = z;
  st->B = B;
  st->H = H;
  st->D = D;
  return LA_OK;
}

la_status lin_attn_state_reset(const la_state* st, void* stream) {
  if (!st || !st->S || !st->z) return LA_ERR_INVALID_ARG;
  size_t heads = (size_t)st->B * st->H;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (heads == 0) return LA_OK;
  if (cudaMemsetAsync(st->S, 0, heads * st->D * st->D * sizeof(float), s) != cudaSuccess ||
      cudaMemsetAsync(st->z, 0, heads * st->D * sizeof(float), s) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  return LA_OK;
}

la_status lin_attn_block_step(const la_params* p, la_state* st, int t_offset, const void* q,
                              const void* k, const void* v, const void* gate, void* out,
                              int commit, void* workspace, size_t workspace_bytes,
                              void* stream) {
  return block_common(p, st, t_offset, q, k, v, gate, out, commit, workspace, workspace_bytes,
                      stream, true);
}

la_status lin_attn_state_update(const la_params* p, la_state* st, int t_offset, const void* k,
                                const void* v, void* workspace, size_t workspace_bytes,
                                void* stream) {
  return block_common(p, st, t_offset, nullptr, k, v, nullptr, nullptr, 1, workspace,
                      workspace_bytes, stream, false);
}

la_status lin_attn_device_status(void* workspace, void* stream) {
  if (!workspace) return LA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int flag = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess ||
      cudaMemcpy(&flag, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  if (flag != 0) {
    // a kernel that gave up may also have left arrival counters behind
    if (cudaMemset(workspace, 0, LA_WORKSPACE_CONTROL_BYTES) != cudaSuccess) {
      cudaGetLastError();
      return LA_ERR_CUDA;
    }
    return LA_ERR_DEVICE_TIMEOUT;
  }
  return LA_OK;
}

const char* lin_attn_status_string(la_status s) {
  switch (s) {
    case LA_OK: return "ok";
    case LA_ERR_INVALID_ARG: return "invalid argument";
    case LA_ERR_UNSUPPORTED: return "unsupported configuration";
    case LA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case LA_ERR_CUDA: return "CUDA runtime error";
    case LA_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
  }
  return "unknown status";
}

int lin_attn_uses_tensor_cores(const la_params* p) {
  if (check_params(p, false) != LA_OK) return 0;
  return want_tc(p, false) ? 1 : 0;
}

}  // extern "C"

/*
 * oracle.c -- plain fp64 CPU reference for ReLU linear attention with 3D RoPE.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the CPU-baseline
 * leg of the benchmark load this library; the product path (the CUDA library
 * and its Python binding) never does. It shares no code, header or table with
 * the CUDA path.
 *
 * What it follows ("SANA-Video: Efficient Video Generation with Block Linear
 * Diffusion Transformer", paper-graph analysis page, section 3.4 "Linear DiT
 * Architecture" and "Block Linear Attention with Constant-Memory KV Cache"):
 *   - ReLU linear attention (the unnumbered equation of "ReLU Linear Attention
 *     Mechanism"): O_i = phi(Q_i) (sum_j phi(K_j)^T V_j) / phi(Q_i) (sum_j
 *     phi(K_j)^T), phi = ReLU, the two sums computed once for all i.
 *   - Eq. 2 ("Integration of 3D Rotary Position Embeddings"): RoPE is applied
 *     after the ReLU, to both phi(Q_i) and phi(K_j) in the numerator; the
 *     denominator keeps the un-rotated phi(Q_i) . sum_j phi(K_j).
 *   - Eq. 3 and the accumulator updates under it: the causal form carries
 *     sum_j phi(K_j)^T V_j (D x D) and sum_j phi(K_j) (D) and adds each new
 *     token's contribution.
 *   - Algorithm 1: a block of frames is denoised against the cached state
 *     and its own tokens; the cache is updated once, after the block.
 *
 * Readings taken where the pages are silent (each is repeated at the code):
 *   - eps: den = phi(q).z + eps, eps added after the dot product.
 *   - RoPE: the D dims are split into three contiguous segments for the
 *     (t, h, w) axes in that order; inside a segment of width d, dims
 *     (2m, 2m+1) form a pair rotated by angle pos * theta^(-2m/d),
 *     (x, y) -> (x cos a - y sin a, x sin a + y cos a); integer positions from 0.
 *   - token order: n = (t*Hg + h)*Wg + w; t = t_offset + n / (Hg*Wg).
 *   - block-causal: a token of block b sees its whole block and all earlier
 *     blocks; positions stay global.
 *   - gate: out <- sigmoid(g) * out elementwise, after the normalisation.
 *
 * All sums run in index order in fp64. Inputs are fp32 arrays holding the
 * values in I/O precision (bf16-rounded values are exact in fp32); they are
 * read as fp64.
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { ORC_BIDIRECTIONAL = 0, ORC_BLOCK_CAUSAL = 1, ORC_TOKEN_CAUSAL = 2 };

typedef struct {
  int B, H, N, D;
  int mode;          /* ORC_BIDIRECTIONAL, ORC_BLOCK_CAUSAL, ORC_TOKEN_CAUSAL */
  int block_tokens;  /* block size for ORC_BLOCK_CAUSAL */
  int rope;          /* 0: no rotation */
  int grid_t, grid_h, grid_w;
  int rope_dt, rope_dh, rope_dw;
  int t_offset;      /* latent frame index of token 0 */
  double theta;
  double eps;
} orc_params;

#define ORC_OK 0
#define ORC_BAD_ARGS (-1)
#define ORC_NO_MEMORY (-2)

int orc_check(const orc_params* p) {
  if (!p) return ORC_BAD_ARGS;
  if (p->B < 0 || p->H < 0 || p->N < 0 || p->D < 1) return ORC_BAD_ARGS;
  if (p->mode < ORC_BIDIRECTIONAL || p->mode > ORC_TOKEN_CAUSAL) return ORC_BAD_ARGS;
  if (p->mode == ORC_BLOCK_CAUSAL &&
      (p->block_tokens <= 0 || p->N % p->block_tokens != 0)) return ORC_BAD_ARGS;
  if (!(p->eps >= 0.0)) return ORC_BAD_ARGS;
  if (p->rope) {
    if (p->rope_dt < 0 || p->rope_dh < 0 || p->rope_dw < 0) return ORC_BAD_ARGS;
    if (p->rope_dt % 2 || p->rope_dh % 2 || p->rope_dw % 2) return ORC_BAD_ARGS;
    if (p->rope_dt + p->rope_dh + p->rope_dw != p->D) return ORC_BAD_ARGS;
    if (p->grid_t < 1 || p->grid_h < 1 || p->grid_w < 1) return ORC_BAD_ARGS;
    if ((long)p->grid_t * p->grid_h * p->grid_w != (long)p->N) return ORC_BAD_ARGS;
    if (!(p->theta > 0.0)) return ORC_BAD_ARGS;
  }
  return ORC_OK;
}

/* phi = ReLU, applied elementwise ("ReLU Linear Attention Mechanism"). */
static double relu(double x) { return x > 0.0 ? x : 0.0; }

/* 3D rotary embedding of one D-vector x at token n, written to y (Eq. 2's
 * RoPE(.)). Axis segments t | h | w over the D dims, adjacent pairs, angle
 * pos_axis * theta^(-2m/d_axis). With rope off, y = x. */
static void rope_rotate(const orc_params* p, long n, const double* x, double* y) {
  int D = p->D;
  if (!p->rope) {
    memcpy(y, x, (size_t)D * sizeof(double));
    return;
  }
  long hw = (long)p->grid_h * p->grid_w;
  long pos[3];
  pos[0] = (long)p->t_offset + n / hw;
  pos[1] = (n / p->grid_w) % p->grid_h;
  pos[2] = n % p->grid_w;
  int width[3] = {p->rope_dt, p->rope_dh, p->rope_dw};
  int base = 0;
  for (int axis = 0; axis < 3; ++axis) {
    int d = width[axis];
    for (int m = 0; m < d / 2; ++m) {
      double inv_freq = pow(p->theta, -2.0 * (double)m / (double)d);
      double angle = (double)pos[axis] * inv_freq;
      double c = cos(angle), s = sin(angle);
      double x0 = x[base + 2 * m], x1 = x[base + 2 * m + 1];
      y[base + 2 * m] = x0 * c - x1 * s;
      y[base + 2 * m + 1] = x0 * s + x1 * c;
    }
    base += d;
  }
}

/* Exported for the RoPE pins: rotate one D-vector x at token n. */
int orc_rope(const orc_params* p, long n, const double* x, double* y) {
  if (!p || !x || !y || p->D < 1) return ORC_BAD_ARGS;
  if (p->rope) {
    if (p->rope_dt % 2 || p->rope_dh % 2 || p->rope_dw % 2) return ORC_BAD_ARGS;
    if (p->rope_dt + p->rope_dh + p->rope_dw != p->D) return ORC_BAD_ARGS;
    if (p->grid_h < 1 || p->grid_w < 1) return ORC_BAD_ARGS;
  }
  rope_rotate(p, n, x, y);
  return ORC_OK;
}

/* ---- per-token building blocks ------------------------------------------ */

/* For token j of one head: phi(k_j) and RoPE(phi(k_j)). */
static void key_features(const orc_params* p, const float* k_head, long j,
                         double* kphi, double* kr) {
  int D = p->D;
  for (int a = 0; a < D; ++a) kphi[a] = relu((double)k_head[(size_t)j * D + a]);
  rope_rotate(p, j, kphi, kr);
}

/* State update of Eq. 3: S += RoPE(phi(k_j))^T v_j, z += phi(k_j). */
static void accumulate(int D, const double* kphi, const double* kr,
                       const float* v_row, double* S, double* z) {
  for (int a = 0; a < D; ++a) {
    for (int c = 0; c < D; ++c) S[(size_t)a * D + c] += kr[a] * (double)v_row[c];
    z[a] += kphi[a];
  }
}

/* One output row with Eq. 2: num = RoPE(phi(q_i)) S, den = phi(q_i) . z + eps,
 * out = num / den, then the gate out *= sigmoid(g). */
static void emit_row(const orc_params* p, const float* q_head, const float* g_head,
                     long i, const double* S, const double* z, double* qphi,
                     double* qr, double* out_row) {
  int D = p->D;
  for (int a = 0; a < D; ++a) qphi[a] = relu((double)q_head[(size_t)i * D + a]);
  rope_rotate(p, i, qphi, qr);
  double den = 0.0;
  for (int a = 0; a < D; ++a) den += qphi[a] * z[a];
  den += p->eps;
  for (int c = 0; c < D; ++c) {
    double num = 0.0;
    for (int a = 0; a < D; ++a) num += qr[a] * S[(size_t)a * D + c];
    double o = num / den;
    if (g_head) {
      double gl = (double)g_head[(size_t)i * D + c];
      o *= 1.0 / (1.0 + exp(-gl));
    }
    out_row[c] = o;
  }
}

/* ---- thread pool over (b, h) ------------------------------------------- */

typedef void (*head_fn)(void* ctx, long bh);

typedef struct {
  head_fn fn;
  void* ctx;
  long count;
  long next;
  int status;
} pool_job;

static void* pool_worker(void* arg) {
  pool_job* job = (pool_job*)arg;
  for (;;) {
    long bh = __atomic_fetch_add(&job->next, 1, __ATOMIC_RELAXED);
    if (bh >= job->count) break;
    job->fn(job->ctx, bh);
  }
  return NULL;
}

int orc_resolve_threads(int nthreads) {
  if (nthreads > 0) return nthreads;
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

static void run_heads(head_fn fn, void* ctx, long count, int nthreads) {
  pool_job job = {fn, ctx, count, 0, 0};
  int nt = orc_resolve_threads(nthreads);
  if (nt > count) nt = (int)(count > 0 ? count : 1);
  if (nt <= 1) {
    pool_worker(&job);
    return;
  }
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nt);
  int started = 0;
  for (int t = 0; t < nt; ++t)
    if (pthread_create(&th[t], NULL, pool_worker, &job) == 0) ++started;
  if (started == 0) pool_worker(&job);
  for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
  free(th);
}

/* ---- full forward -------------------------------------------------------- */

typedef struct {
  const orc_params* p;
  const float *q, *k, *v, *g;
  const double *S0, *z0;
  double *out, *S_final, *z_final;
  int failed;
} fwd_ctx;

static void forward_head(void* vctx, long bh) {
  fwd_ctx* c = (fwd_ctx*)vctx;
  const orc_params* p = c->p;
  int D = p->D;
  long N = p->N;
  size_t off = (size_t)bh * (size_t)N * D;
  const float* qh = c->q + off;
  const float* kh = c->k + off;
  const float* vh = c->v + off;
  const float* gh = c->g ? c->g + off : NULL;
  double* oh = c->out ? c->out + off : NULL;

  double* S = (double*)calloc((size_t)D * D, sizeof(double));
  double* Sblk = (double*)calloc((size_t)D * D, sizeof(double));
  double* Sap = (double*)calloc((size_t)D * D, sizeof(double));
  double* z = (double*)calloc((size_t)D, sizeof(double));
  double* zblk = (double*)calloc((size_t)D, sizeof(double));
  double* zap = (double*)calloc((size_t)D, sizeof(double));
  double* t0 = (double*)malloc((size_t)D * sizeof(double));
  double* t1 = (double*)malloc((size_t)D * sizeof(double));
  if (!S || !Sblk || !Sap || !z || !zblk || !zap || !t0 || !t1) {
    __atomic_store_n(&c->failed, 1, __ATOMIC_RELAXED);
    goto done;
  }
  if (c->S0) memcpy(S, c->S0 + (size_t)bh * D * D, (size_t)D * D * sizeof(double));
  if (c->z0) memcpy(z, c->z0 + (size_t)bh * D, (size_t)D * sizeof(double));

  if (p->mode == ORC_BIDIRECTIONAL) {
    /* The two accumulators over all N tokens, then every output row. */
    for (long j = 0; j < N; ++j) {
      key_features(p, kh, j, t0, t1);
      accumulate(D, t0, t1, vh + (size_t)j * D, S, z);
    }
    if (oh)
      for (long i = 0; i < N; ++i) emit_row(p, qh, gh, i, S, z, t0, t1, oh + (size_t)i * D);
  } else if (p->mode == ORC_BLOCK_CAUSAL) {
    /* Algorithm 1 per block: the block's own state, the outputs against
     * (carried state + block state), then the carried state takes the block. */
    long bt = p->block_tokens;
    for (long b0 = 0; b0 < N; b0 += bt) {
      memset(Sblk, 0, (size_t)D * D * sizeof(double));
      memset(zblk, 0, (size_t)D * sizeof(double));
      for (long j = b0; j < b0 + bt; ++j) {
        key_features(p, kh, j, t0, t1);
        accumulate(D, t0, t1, vh + (size_t)j * D, Sblk, zblk);
      }
      for (size_t e = 0; e < (size_t)D * D; ++e) Sap[e] = S[e] + Sblk[e];
      for (int a = 0; a < D; ++a) zap[a] = z[a] + zblk[a];
      if (oh)
        for (long i = b0; i < b0 + bt; ++i)
          emit_row(p, qh, gh, i, Sap, zap, t0, t1, oh + (size_t)i * D);
      for (size_t e = 0; e < (size_t)D * D; ++e) S[e] = S[e] + Sblk[e];
      for (int a = 0; a < D; ++a) z[a] = z[a] + zblk[a];
    }
  } else {
    /* Eq. 3: token i sees tokens j <= i; add token i, then emit row i. */
    for (long i = 0; i < N; ++i) {
      key_features(p, kh, i, t0, t1);
      accumulate(D, t0, t1, vh + (size_t)i * D, S, z);
      if (oh) emit_row(p, qh, gh, i, S, z, t0, t1, oh + (size_t)i * D);
    }
  }
  if (c->S_final) memcpy(c->S_final + (size_t)bh * D * D, S, (size_t)D * D * sizeof(double));
  if (c->z_final) memcpy(c->z_final + (size_t)bh * D, z, (size_t)D * sizeof(double));
done:
  free(S); free(Sblk); free(Sap); free(z); free(zblk); free(zap); free(t0); free(t1);
}

/* Full output [B,H,N,D] in fp64. S0/z0 (nullable, [B,H,D,D] / [B,H,D]) is a
 * carried state that the causal modes start from; S_final/z_final (nullable)
 * receive the state after the last token (for ORC_BIDIRECTIONAL: the sums
 * over all tokens, plus S0/z0 if given). */
int orc_forward(const orc_params* p, const float* q, const float* k, const float* v,
                const float* g, const double* S0, const double* z0, double* out,
                double* S_final, double* z_final, int nthreads) {
  int rc = orc_check(p);
  if (rc) return rc;
  long heads = (long)p->B * p->H;
  if (heads == 0 || p->N == 0) return ORC_OK;
  if (!k || !v || (out && !q)) return ORC_BAD_ARGS;
  fwd_ctx c = {p, q, k, v, g, S0, z0, out, S_final, z_final, 0};
  run_heads(forward_head, &c, heads, nthreads);
  return c.failed ? ORC_NO_MEMORY : ORC_OK;
}

/* ---- sampled rows --------------------------------------------------------- */

typedef struct {
  const orc_params* p;
  const float *q, *k, *v, *g;
  const double *S0, *z0;
  const long long* rows;   /* flattened (b*H + h)*N + n */
  long nrows;
  double* out_rows;        /* [nrows][D] */
  long* order;             /* row indices sorted by flattened index */
  long* head_start;        /* [heads + 1] offsets into order */
  int failed;
} rows_ctx;

static int cmp_rows(const void* a, const void* b, void* arg) {
  const long long* rows = (const long long*)arg;
  long long ra = rows[*(const long*)a], rb = rows[*(const long*)b];
  return (ra > rb) - (ra < rb);
}

static void rows_head(void* vctx, long bh) {
  rows_ctx* c = (rows_ctx*)vctx;
  const orc_params* p = c->p;
  long lo = c->head_start[bh], hi = c->head_start[bh + 1];
  if (lo == hi) return;
  int D = p->D;
  long N = p->N;
  size_t off = (size_t)bh * (size_t)N * D;
  const float* qh = c->q + off;
  const float* kh = c->k + off;
  const float* vh = c->v + off;
  const float* gh = c->g ? c->g + off : NULL;
  double* S = (double*)calloc((size_t)D * D, sizeof(double));
  double* Sblk = (double*)calloc((size_t)D * D, sizeof(double));
  double* Sap = (double*)calloc((size_t)D * D, sizeof(double));
  double* z = (double*)calloc((size_t)D, sizeof(double));
  double* zblk = (double*)calloc((size_t)D, sizeof(double));
  double* zap = (double*)calloc((size_t)D, sizeof(double));
  double* t0 = (double*)malloc((size_t)D * sizeof(double));
  double* t1 = (double*)malloc((size_t)D * sizeof(double));
  if (!S || !Sblk || !Sap || !z || !zblk || !zap || !t0 || !t1) {
    __atomic_store_n(&c->failed, 1, __ATOMIC_RELAXED);
    goto done;
  }
  if (c->S0) memcpy(S, c->S0 + (size_t)bh * D * D, (size_t)D * D * sizeof(double));
  if (c->z0) memcpy(z, c->z0 + (size_t)bh * D, (size_t)D * sizeof(double));
  long last_n = (long)(c->rows[c->order[hi - 1]] - (long long)bh * N);
  long r = lo;
  if (p->mode == ORC_BIDIRECTIONAL) {
    for (long j = 0; j < N; ++j) {
      key_features(p, kh, j, t0, t1);
      accumulate(D, t0, t1, vh + (size_t)j * D, S, z);
    }
    for (; r < hi; ++r) {
      long idx = c->order[r];
      long n = (long)(c->rows[idx] - (long long)bh * N);
      emit_row(p, qh, gh, n, S, z, t0, t1, c->out_rows + (size_t)idx * D);
    }
  } else if (p->mode == ORC_BLOCK_CAUSAL) {
    long bt = p->block_tokens;
    for (long b0 = 0; b0 <= last_n; b0 += bt) {
      memset(Sblk, 0, (size_t)D * D * sizeof(double));
      memset(zblk, 0, (size_t)D * sizeof(double));
      for (long j = b0; j < b0 + bt; ++j) {
        key_features(p, kh, j, t0, t1);
        accumulate(D, t0, t1, vh + (size_t)j * D, Sblk, zblk);
      }
      for (size_t e = 0; e < (size_t)D * D; ++e) Sap[e] = S[e] + Sblk[e];
      for (int a = 0; a < D; ++a) zap[a] = z[a] + zblk[a];
      for (; r < hi; ++r) {
        long idx = c->order[r];
        long n = (long)(c->rows[idx] - (long long)bh * N);
        if (n >= b0 + bt) break;
        emit_row(p, qh, gh, n, Sap, zap, t0, t1, c->out_rows + (size_t)idx * D);
      }
      for (size_t e = 0; e < (size_t)D * D; ++e) S[e] = S[e] + Sblk[e];
      for (int a = 0; a < D; ++a) z[a] = z[a] + zblk[a];
    }
  } else {
    for (long i = 0; i <= last_n; ++i) {
      key_features(p, kh, i, t0, t1);
      accumulate(D, t0, t1, vh + (size_t)i * D, S, z);
      for (; r < hi; ++r) {
        long idx = c->order[r];
        long n = (long)(c->rows[idx] - (long long)bh * N);
        if (n != i) break;
        emit_row(p, qh, gh, n, S, z, t0, t1, c->out_rows + (size_t)idx * D);
      }
    }
  }
done:
  free(S); free(Sblk); free(Sap); free(z); free(zblk); free(zap); free(t0); free(t1);
}

/* Output rows only: rows[r] = (b*H + h)*N + n; out_rows is [nrows][D]. Same
 * arithmetic as orc_forward, computing each needed state once per head. */
int orc_forward_rows(const orc_params* p, const float* q, const float* k, const float* v,
                     const float* g, const double* S0, const double* z0,
                     const long long* rows, long nrows, double* out_rows, int nthreads) {
  int rc = orc_check(p);
  if (rc) return rc;
  if (nrows == 0) return ORC_OK;
  if (!q || !k || !v || !rows || !out_rows || nrows < 0) return ORC_BAD_ARGS;
  long heads = (long)p->B * p->H;
  long long total = (long long)heads * p->N;
  for (long r = 0; r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= total) return ORC_BAD_ARGS;
  long* order = (long*)malloc(sizeof(long) * (size_t)nrows);
  long* head_start = (long*)calloc((size_t)heads + 1, sizeof(long));
  if (!order || !head_start) {
    free(order); free(head_start);
    return ORC_NO_MEMORY;
  }
  for (long r = 0; r < nrows; ++r) order[r] = r;
  qsort_r(order, (size_t)nrows, sizeof(long), cmp_rows, (void*)rows);
  for (long r = 0; r < nrows; ++r) head_start[rows[r] / p->N + 1]++;
  for (long h = 0; h < heads; ++h) head_start[h + 1] += head_start[h];
  rows_ctx c = {p, q, k, v, g, S0, z0, rows, nrows, out_rows, order, head_start, 0};
  run_heads(rows_head, &c, heads, nthreads);
  free(order); free(head_start);
  return c.failed ? ORC_NO_MEMORY : ORC_OK;
}

/* ---- state over a token range ---------------------------------------------- */

typedef struct {
  const orc_params* p;
  const float *k, *v;
  long n0, n1;
  double *S, *z;
  int failed;
} state_ctx;

static void state_head(void* vctx, long bh) {
  state_ctx* c = (state_ctx*)vctx;
  const orc_params* p = c->p;
  int D = p->D;
  size_t off = (size_t)bh * (size_t)p->N * D;
  double* S = c->S + (size_t)bh * D * D;
  double* z = c->z + (size_t)bh * D;
  double* t0 = (double*)malloc((size_t)D * sizeof(double));
  double* t1 = (double*)malloc((size_t)D * sizeof(double));
  if (!t0 || !t1) {
    __atomic_store_n(&c->failed, 1, __ATOMIC_RELAXED);
    free(t0); free(t1);
    return;
  }
  memset(S, 0, (size_t)D * D * sizeof(double));
  memset(z, 0, (size_t)D * sizeof(double));
  for (long j = c->n0; j < c->n1; ++j) {
    key_features(p, c->k + off, j, t0, t1);
    accumulate(D, t0, t1, c->v + off + (size_t)j * D, S, z);
  }
  free(t0); free(t1);
}

/* S[bh] = sum_{j in [n0, n1)} RoPE(phi(k_j))^T v_j and z[bh] = sum phi(k_j)
 * for every head: the two accumulators of the linear-attention equation. */
int orc_state(const orc_params* p, const float* k, const float* v, long n0, long n1,
              double* S, double* z, int nthreads) {
  orc_params pp;
  if (!p) return ORC_BAD_ARGS;
  pp = *p;
  pp.mode = ORC_BIDIRECTIONAL;
  int rc = orc_check(&pp);
  if (rc) return rc;
  if (n0 < 0 || n1 < n0 || n1 > p->N || !S || !z) return ORC_BAD_ARGS;
  long heads = (long)p->B * p->H;
  if (heads == 0) return ORC_OK;
  if (!k || !v) return ORC_BAD_ARGS;
  state_ctx c = {&pp, k, v, n0, n1, S, z, 0};
  run_heads(state_head, &c, heads, nthreads);
  return c.failed ? ORC_NO_MEMORY : ORC_OK;
}

/* ---- literal O(N^2) form --------------------------------------------------- */

typedef struct {
  const orc_params* p;
  const float *q, *k, *v, *g;
  double* out;
  int failed;
} brute_ctx;

static void brute_head(void* vctx, long bh) {
  brute_ctx* c = (brute_ctx*)vctx;
  const orc_params* p = c->p;
  int D = p->D;
  long N = p->N;
  size_t off = (size_t)bh * (size_t)N * D;
  double* kphi = (double*)malloc((size_t)N * D * sizeof(double));
  double* kr = (double*)malloc((size_t)N * D * sizeof(double));
  double* qphi = (double*)malloc((size_t)D * sizeof(double));
  double* qr = (double*)malloc((size_t)D * sizeof(double));
  double* num = (double*)malloc((size_t)D * sizeof(double));
  if (!kphi || !kr || !qphi || !qr || !num) {
    __atomic_store_n(&c->failed, 1, __ATOMIC_RELAXED);
    goto done;
  }
  for (long j = 0; j < N; ++j)
    key_features(p, c->k + off, j, kphi + (size_t)j * D, kr + (size_t)j * D);
  for (long i = 0; i < N; ++i) {
    /* scope of token i: all tokens, its block and earlier blocks, or j <= i */
    long jend = N;
    if (p->mode == ORC_BLOCK_CAUSAL) jend = (i / p->block_tokens + 1) * (long)p->block_tokens;
    if (p->mode == ORC_TOKEN_CAUSAL) jend = i + 1;
    for (int a = 0; a < D; ++a) qphi[a] = relu((double)c->q[off + (size_t)i * D + a]);
    rope_rotate(p, i, qphi, qr);
    for (int e = 0; e < D; ++e) num[e] = 0.0;
    double den = 0.0;
    for (long j = 0; j < jend; ++j) {
      /* weight of token j in the numerator: RoPE(phi(q_i)) . RoPE(phi(k_j));
       * in the denominator: phi(q_i) . phi(k_j) (Eq. 2) */
      double wn = 0.0, wd = 0.0;
      for (int a = 0; a < D; ++a) {
        wn += qr[a] * kr[(size_t)j * D + a];
        wd += qphi[a] * kphi[(size_t)j * D + a];
      }
      for (int e = 0; e < D; ++e) num[e] += wn * (double)c->v[off + (size_t)j * D + e];
      den += wd;
    }
    den += p->eps;
    for (int e = 0; e < D; ++e) {
      double o = num[e] / den;
      if (c->g) o *= 1.0 / (1.0 + exp(-(double)c->g[off + (size_t)i * D + e]));
      c->out[off + (size_t)i * D + e] = o;
    }
  }
done:
  free(kphi); free(kr); free(qphi); free(qr); free(num);
}

/* out_i = sum_j (RoPE(phi q_i) . RoPE(phi k_j)) v_j / (sum_j phi q_i . phi k_j + eps)
 * over the scope of each mode: the attention-weight form the factorised
 * equations rewrite. O(N^2 D) -- tiny inputs only. */
int orc_bruteforce(const orc_params* p, const float* q, const float* k, const float* v,
                   const float* g, double* out, int nthreads) {
  int rc = orc_check(p);
  if (rc) return rc;
  long heads = (long)p->B * p->H;
  if (heads == 0 || p->N == 0) return ORC_OK;
  if (!q || !k || !v || !out) return ORC_BAD_ARGS;
  brute_ctx c = {p, q, k, v, g, out, 0};
  run_heads(brute_head, &c, heads, nthreads);
  return c.failed ? ORC_NO_MEMORY : ORC_OK;
}

/*
 * linattn.h -- C ABI of a B200 (sm_100a) library for ReLU linear attention
 * with 3D rotary position embeddings, the token mixer of the SANA-Video
 * linear diffusion transformer.
 *
 * Source of the operation ("SANA-Video: Efficient Video Generation with Block
 * Linear Diffusion Transformer", paper-graph analysis page, section 3.4):
 *   - "ReLU Linear Attention Mechanism" (unnumbered equation): phi = ReLU,
 *     S = sum_j phi(k_j)^T v_j (D x D) and z = sum_j phi(k_j) (D) are built
 *     once and every query reads them.
 *   - "Integration of 3D RoPE", Eq. 2: RoPE is applied after phi, in the
 *     numerator only:
 *         out_i = RoPE(phi(q_i)) . S / (phi(q_i) . z + eps),
 *         S     = sum_j RoPE(phi(k_j))^T v_j,   z = sum_j phi(k_j).
 *   - "Block Linear Attention with Constant-Memory KV Cache", Eq. 3 and
 *     Algorithm 1: the state (S, z) is carried across blocks of frames; a
 *     block reads the cached state plus its own tokens, and the cache is
 *     updated once, after the block.
 *   - The SANA-Video 2.0 pages (neuraltrendhub summary and abstract) call the
 *     layers "gated" linear attention without a formula; the gate taken here
 *     is out_i <- sigmoid(g_i) * out_i elementwise, after the normalisation.
 *
 * Readings where the pages say nothing (also listed in the design notes):
 *   RoPE: the D dims split into three contiguous segments (t | h | w) of widths
 *   rope_dt, rope_dh, rope_dw; inside a segment of width d, dims (2m, 2m+1)
 *   rotate by pos * theta^(-2m/d): (x, y) -> (x cos a - y sin a,
 *   x sin a + y cos a). Token n of a head sits at t = t_offset + n/(Hg*Wg),
 *   h = (n/Wg) % Hg, w = n % Wg. eps is added after the dot product, so a row
 *   with phi(q_i) = 0 yields 0.
 *
 * Conventions for every entry point:
 *   - Memory. The caller owns all device memory (inputs, output, state,
 *     workspace); the library allocates and frees nothing. Calls are
 *     re-entrant: the library's process-wide state is a mutex-guarded record
 *     of the kernels whose shared-memory limit it has set on each device, and
 *     the one device array shared by all calls of lin_attn_forward_noalloc
 *     (see its comment).
 *   - Layout. q, k, v, gate, out are contiguous [B, H, N, D] (or [B, N, H, D]
 *     with p->layout = LA_LAYOUT_BNHD) with D innermost, in the I/O dtype.
 *     The state is fp32: S [B, H, D, D] with
 *     S[a][c] = sum_j RoPE(phi(k_j))_a v_j,c, and z [B, H, D].
 *   - Asynchrony. A call checks its arguments on the host, enqueues kernels on
 *     `stream` (a cudaStream_t passed as void*, NULL = legacy default stream)
 *     and returns; results are valid once the stream reaches that point. The
 *     tensor-core kernels use programmatic dependent launch: each may start
 *     behind the kernel before it on the stream, but reads its inputs and
 *     writes memory only after that kernel has completed.
 *   - Errors. Every call returns la_status; nothing aborts, prints or throws.
 *     Invalid arguments are rejected before any launch and leave memory
 *     untouched. A launch failure returns LA_ERR_CUDA.
 *   - Alignment. Every tensor pointer and the workspace must be 16-byte
 *     aligned; D * sizeof(dtype) is then a multiple of 16.
 *   - Aliasing. out may not overlap q, k, v or gate.
 *   - Determinism. Reductions run in a fixed order: the same inputs on the
 *     same device give bit-identical outputs and state.
 */
#ifndef LINATTN_H
#define LINATTN_H

#include <stddef.h>

#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LA_OK = 0,
  LA_ERR_INVALID_ARG = 1,  /* a pointer, size or field is out of range */
  LA_ERR_UNSUPPORTED = 2,  /* valid, but outside what the kernels handle */
  LA_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small */
  LA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  LA_ERR_DEVICE_TIMEOUT = 5 /* a kernel gave up a bounded wait (see
                               lin_attn_device_status) */
} la_status;

typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;   /* I/O dtype; state is fp32 */

typedef enum { LA_BIDIRECTIONAL = 0, LA_BLOCK_CAUSAL = 1, LA_TOKEN_CAUSAL = 2 } la_mode;

/* Memory order of q, k, v, gate and out (D innermost either way). BNHD is
 * the order a fused QKV projection of [B, N, C] hidden states writes its
 * heads in, so the op reads it without a transpose. */
typedef enum { LA_LAYOUT_BHND = 0, LA_LAYOUT_BNHD = 1 } la_layout;

typedef struct {
  int B, H, N, D;        /* batch, heads, tokens per head, head dim.
                            D in {32, 64, 112, 128} (112: the SANA-Video 2B
                            head dim; bf16 forwards run it on the 128-wide
                            tensor-core kernels with zero padding, block steps
                            on the CUDA-core kernels); N >= 0 (N = 0: no
                            work). */
  la_dtype dtype;        /* dtype of q, k, v, gate and out */
  la_mode mode;          /* bidirectional, block-causal or token-causal */
  int block_tokens;      /* block-causal: tokens per block, N % block_tokens == 0.
                            A token of block b sees blocks 0..b (its own block
                            whole). Ignored in the other modes. */
  int rope;              /* 0: no rotation (then the grid fields are ignored) */
  int grid_t, grid_h, grid_w;     /* latent grid; N == grid_t*grid_h*grid_w */
  int rope_dt, rope_dh, rope_dw;  /* even widths with sum D (t, h, w order) */
  double rope_theta;     /* RoPE base, > 0 (10000 in the workloads here) */
  float eps;             /* added to the denominator, >= 0 (1e-6 here) */
  la_layout layout;      /* LA_LAYOUT_BHND ([B,H,N,D], zero) or LA_LAYOUT_BNHD
                            ([B,N,H,D]); every tensor of the call uses it, and
                            a block step's q, k, v, gate, out are [B,N,H,D]
                            with N the block's tokens */
} la_params;

/* A carried block-causal state: caller-owned device memory, fp32,
 * S [B, H, D, D] and z [B, H, D] (16-byte aligned). */
typedef struct {
  float* S;
  float* z;
  int B, H, D;
} la_state;

/* Size of the control block at the start of every workspace (included in the
 * sizes below): a flag word and one arrival counter per segment, zero
 * between calls. */
#define LA_WORKSPACE_CONTROL_BYTES 65536u

/* Bytes of workspace lin_attn_forward needs for `p` on the current device
 * (the size depends on the device's SM count). Writes *bytes; no launch. */
LA_API la_status lin_attn_workspace_size(const la_params* p, size_t* bytes);

/* Bytes of workspace lin_attn_block_step / lin_attn_state_update need for a
 * block of p->N tokens (mode and block_tokens are ignored). */
LA_API la_status lin_attn_block_step_workspace_size(const la_params* p, size_t* bytes);

/* The whole-sequence forward (Eq. 2, plus the gate when gate != NULL).
 *   bidirectional: out_i uses S, z summed over all N tokens of its head.
 *   block-causal:  out_i of block b uses S, z summed over blocks 0..b, which
 *                  is Algorithm 1 run with an empty initial cache.
 *   token-causal:  out_i uses S, z summed over tokens 0..i of its head (the
 *                  causal form, Eq. 3 of "Block Linear Attention with
 *                  Constant-Memory KV Cache"). bf16 at D = 64 (RoPE
 *                  widths multiples of 8) runs on the tensor cores: each
 *                  CTA starts from the sums over the tokens before its
 *                  range and walks it in chunks of 128 tokens, adding the
 *                  masked in-chunk products and carrying the state. Other
 *                  shapes run on the CUDA-core kernels in chunks of 32.
 * q, k, v, out: [B,H,N,D] device pointers in p->dtype. gate: NULL or the same
 * shape and dtype (logits; out is multiplied by their sigmoid).
 * workspace: device memory of at least lin_attn_workspace_size bytes, 256-byte
 * aligned. Its first LA_WORKSPACE_CONTROL_BYTES bytes are a control block (an
 * error flag and per-segment arrival counters) that must be zero before the
 * first call that uses the workspace -- allocate it zeroed; every call leaves
 * the block zero, and lin_attn_device_status re-zeroes it after a call that
 * gave up a bounded wait. The rest of the workspace may hold anything on entry
 * and is clobbered.
 * Limits (else LA_ERR_UNSUPPORTED, nothing launched): B * H <= 2^24, and
 * B * H times the segments of a head (1 bidirectional, N / block_tokens
 * block-causal, ceil(N / 32) token-causal) <= INT_MAX.
 * Returns LA_OK once the work is enqueued on `stream`. */
LA_API la_status lin_attn_forward(const la_params* p, const void* q, const void* k,
                           const void* v, const void* gate, void* out,
                           void* workspace, size_t workspace_bytes, void* stream);

/* lin_attn_forward that also records four caller-created CUDA events (as
 * void*, e.g. cudaEvent_t) on `stream`: events[0] before the state build,
 * events[1] after it, events[2] after the reduction (at once when the state
 * build performs it), events[3] after the apply step, so a caller can time
 * each kernel on the launching stream.
 * events may be NULL (then this is lin_attn_forward). */
LA_API la_status lin_attn_forward_timed(const la_params* p, const void* q, const void* k,
                                        const void* v, const void* gate, void* out,
                                        void* workspace, size_t workspace_bytes, void* stream,
                                        void* const* events);

/* Linear cross-attention: the p->N queries of each (b, h) read S, z summed
 * over n_kv keys and values of the same (b, h), e.g. video tokens attending
 * to text tokens (the linear cross-attention the SANA-Video paper-graph page
 * lists beside self-attention):
 *     out_i = phi(q_i) . S / (phi(q_i) . z + eps) (* sigmoid(g_i)),
 *     S = sum_j phi(k_j)^T v_j,   z = sum_j phi(k_j),   j < n_kv.
 * q, gate, out: [B,H,N,D]; k, v: [B,H,n_kv,D], all in p->dtype. The two
 * sequences share no positions: p->rope must be 0 and p->mode bidirectional
 * (else LA_ERR_INVALID_ARG); n_kv >= 1 (N = 0: no work).
 * workspace: at least lin_attn_cross_workspace_size bytes, as in
 * lin_attn_forward. */
LA_API la_status lin_attn_cross_forward(const la_params* p, int n_kv, const void* q,
                                        const void* k, const void* v, const void* gate,
                                        void* out, void* workspace, size_t workspace_bytes,
                                        void* stream);

/* Bytes of workspace lin_attn_cross_forward needs for `p` and n_kv. */
LA_API la_status lin_attn_cross_workspace_size(const la_params* p, int n_kv, size_t* bytes);

/* Size of the fixed scratch area that lin_attn_forward_noalloc uses. */
#define LA_NOALLOC_SCRATCH_BYTES (32u << 20)

/* lin_attn_forward for callers that cannot allocate device memory for a
 * workspace -- for example a plugin inside a host engine that owns all device
 * memory through a pre-planned arena and forbids extra allocations, or a
 * real-time generation loop that must never call cudaMalloc (which can
 * synchronise the device). The paper has no counterpart: this is a packaging
 * choice of the library, not a step of the method.
 *
 * Instead of a caller workspace it uses one file-scope device array of
 * LA_NOALLOC_SCRATCH_BYTES (32 MiB) inside the library. Every GPU on which the
 * library is loaded holds that array until the process exits. The call itself
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   - Set-up: the first call on a device (with that device current) looks up
 *     the array's device address once; make that first call before any stream
 *     capture.
 *   - Limit: a problem whose workspace (lin_attn_workspace_size) exceeds
 *     LA_NOALLOC_SCRATCH_BYTES is rejected with LA_ERR_WORKSPACE before any
 *     launch.
 *   - Sharing: all calls on a device share the one array, and it keeps the
 *     last call's contents (the call clears what must start at zero). Calls
 *     that overlap on the GPU -- on different streams, or from different host
 *     threads without ordering -- race on it and give wrong results; order them
 *     on one stream.
 *   - No status query: the array's control block (with the flag a kernel sets
 *     when it gives up a bounded wait) is cleared at the start of every call,
 *     and no entry point reads it back, so a call whose kernel gave up such a
 *     wait cannot be detected on this path. Callers that need that check use
 *     lin_attn_forward with lin_attn_device_status.
 * Arguments and results are those of lin_attn_forward without the workspace. */
LA_API la_status lin_attn_forward_noalloc(const la_params* p, const void* q, const void* k,
                                          const void* v, const void* gate, void* out,
                                          void* stream);

/* Wrap caller-owned state buffers (no allocation, no launch). S and z must
 * be device pointers, 16-byte aligned, of [B,H,D,D] and [B,H,D] floats. */
LA_API la_status lin_attn_state_init(la_state* st, int B, int H, int D, float* S, float* z);

/* Zero the state asynchronously on `stream` (the empty cache of Algorithm 1). */
LA_API la_status lin_attn_state_reset(const la_state* st, void* stream);

/* One block of Algorithm 1. p->N is the number of tokens in this block (its
 * frames are grid_t latent frames starting at global frame t_offset, so RoPE
 * positions stay global); p->mode and p->block_tokens are ignored.
 *   out_i = RoPE(phi(q_i)) (S + S_blk) / (phi(q_i) . (z + z_blk) + eps)
 * with (S, z) the carried state and (S_blk, z_blk) the sums over this block.
 * commit != 0 then sets S += S_blk, z += z_blk in place (the cache update at
 * the last denoising step); commit == 0 leaves the state byte-identical.
 * gate may be NULL. The state must match p (B, H, D). q, k, v, gate and out
 * may not share bytes with S or z, nor S with z (else LA_ERR_INVALID_ARG,
 * nothing launched): the state is updated in place while they are read. */
LA_API la_status lin_attn_block_step(const la_params* p, la_state* st, int t_offset,
                              const void* q, const void* k, const void* v,
                              const void* gate, void* out, int commit,
                              void* workspace, size_t workspace_bytes, void* stream);

/* The cache update alone (Algorithm 1's G^KV step, from the clean latent's
 * k and v): S += sum_j RoPE(phi(k_j))^T v_j, z += sum_j phi(k_j) over the
 * p->N tokens of the block. Same arguments as lin_attn_block_step without
 * q, gate and out. */
LA_API la_status lin_attn_state_update(const la_params* p, la_state* st, int t_offset,
                                const void* k, const void* v, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Synchronise `stream` and report whether any kernel of the last calls that
 * used `workspace` gave up a bounded wait (LA_ERR_DEVICE_TIMEOUT) -- a safety
 * net that should never fire. Then re-zeroes the control block. */
LA_API la_status lin_attn_device_status(void* workspace, void* stream);

/* Static description of a status code. */
LA_API const char* lin_attn_status_string(la_status s);

/* Which kernel family lin_attn_forward would use for `p` on the current
 * device: 1 = tensor-core (tcgen05 + TMA, bf16 I/O, D in {64, 112, 128}),
 * 0 = CUDA-core (fp32 I/O, token-causal mode other than bf16 at D = 64,
 * or shapes outside the tensor-core path). */
LA_API int lin_attn_uses_tensor_cores(const la_params* p);

/* ---- Mix-FFN temporal convolution with the last-frame cache -------------
 * The temporal convolution of the spatial-temporal Mix-FFN (SANA-Video
 * paper-graph page, "Spatial-Temporal Mix-FFN": kernel size 3 along time, a
 * 3x1x1 kernel on the [T, H, W, C] hidden states, added through a shortcut)
 * and its block-causal form ("Block Causal Mix-FFN": a zero frame after the
 * block, the previous block's last frame cached and put before it; the conv
 * cache of Algorithm 1). Per channel c (depthwise), frame t, position s:
 *     y[b,t,s,c] = x[b,t,s,c] + w[0][c] x[b,t-1,s,c] + w[1][c] x[b,t,s,c]
 *                  + w[2][c] x[b,t+1,s,c]  (+ bias[c]),
 * with frame T (after the block) zero and frame -1 = cache_in, or zero when
 * cache_in is NULL (the first block, or a whole-sequence call).
 *   x, y:      [B, T, S, C] in dtype, C innermost (the [B, N, C] hidden states
 *              of a DiT block, N = T * S, S = grid_h * grid_w).
 *   weight:    fp32 [3][C], tap 0 on frame t-1, tap 1 on t, tap 2 on t+1.
 *   bias:      fp32 [C], or NULL (none).
 *   cache_in:  [B, S, C] in dtype, or NULL.
 *   cache_out: [B, S, C] in dtype, or NULL; receives x[:, T-1], the block's
 *              last input frame, after cache_in has been read, so cache_out ==
 *              cache_in updates the cache in place.
 * Arithmetic in fp32, one rounding to dtype per output; no workspace.
 * Errors (LA_ERR_INVALID_ARG, nothing launched): a negative size; dtype not
 * LA_F32 / LA_BF16; C not a multiple of 16 bytes' worth of dtype (8 bf16,
 * 4 fp32); x, y or weight NULL when there is work; any pointer not 16-byte
 * aligned; y overlapping another buffer; cache_out overlapping x, weight or
 * bias, or overlapping cache_in without being equal to it. B*T*S*C = 0: no
 * work, cache_out untouched. */
LA_API la_status lin_attn_temporal_conv(int B, int T, int S, int C, la_dtype dtype,
                                        const void* x, const float* weight, const float* bias,
                                        const void* cache_in, void* y, void* cache_out,
                                        void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LINATTN_H */

/*
 * hsa.h - C ABI of the Heterogeneous Step Allocation (HSA) denoising step on
 * NVIDIA B200 (sm_100a).  Implemented by libhsa.so.
 *
 * The method ("Not All Tokens Need 40 Steps: Heterogeneous Step Allocation in
 * Diffusion Transformers for Efficient Video Generation"; its steps are laid
 * out in "Technical Summary: Heterogeneous Step Allocation (HSA) for
 * Efficient Video Generation", sections 2.1-2.4, cited below as [TS]) splits
 * the N tokens of a video latent into K groups with step budgets s_k | T.
 * Only the tokens active at a global iteration run through the transformer;
 * their fresh K/V rows overwrite a per-layer KV cache that every active query
 * attends to in full; and one cached Euler update advances all N tokens.
 *
 * Conventions for every call:
 *  - Pointers marked (device) are caller-owned device memory on the device
 *    that was current at hsa_create; (host) pointers are host memory.  All
 *    device pointers must be 16-byte aligned.  Tensors are dense row-major
 *    with exactly the strides given.
 *  - bf16 buffers are passed as void* and hold IEEE bfloat16 values.
 *  - Every call enqueues its kernels on the context's stream and returns
 *    without waiting for them; the caller orders other work on that stream.
 *    A context is not re-entrant: calls on one context must not overlap.
 *  - Calls return a status and never abort.  A status other than HSA_OK comes
 *    with a message from hsa_last_error().  Argument errors are detected on
 *    the host before anything is launched.  Errors found by kernels (an index
 *    out of range, a wait that timed out) set a device flag that
 *    hsa_sync_check() reads.
 *  - Shapes: C = 16 latent channels; head_dim d = D / H is 64 or 128;
 *    D % 128 == 0; F % 64 == 0; 1 <= N < 2^31; 1 <= K <= 8.
 */
#ifndef HSA_H_
#define HSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSA_OK = 0,
  HSA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, n out of range, ... */
  HSA_ERR_BUDGET = 2,       /* s_k does not divide T, s_1 != T, counts do not sum to N */
  HSA_ERR_SHAPE = 3,        /* model shape outside the supported set above */
  HSA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  HSA_ERR_OOM = 5,          /* scratch allocation failed in hsa_create */
  HSA_ERR_TIMEOUT = 6,      /* a kernel's bounded wait expired (read by hsa_sync_check) */
  HSA_ERR_DEVICE_CHECK = 7, /* a kernel found a bad index or a NaN score (hsa_sync_check) */
  HSA_ERR_SCRATCH_LIMIT = 8 /* a size beyond the fixed scratch of hsa_select_groups_static */
} hsa_status;

/* Model shape.  N tokens, C latent channels, D hidden, H heads, F MLP width, L layers. */
typedef struct {
  int N, C, D, H, F, L;
} hsa_model_cfg;

/* One transformer block's weights, bf16, Linear layout [out, in], row-major (device). */
typedef struct {
  const void* w_qkv; /* [3D, D]: rows 0..D-1 -> Q, D..2D-1 -> K, 2D..3D-1 -> V */
  const void* w_o;   /* [D, D] */
  const void* w_1;   /* [F, D] */
  const void* w_2;   /* [D, F] */
} hsa_layer_weights;

/* Whole-model weights for hsa_step. */
typedef struct {
  const float* w_in;               /* fp32 [D, C] latent -> hidden embed (device) */
  const float* w_head;             /* fp32 [C, D] hidden -> velocity head (device) */
  const hsa_layer_weights* layers; /* host array of L blocks */
} hsa_model_weights;

/* Per-loop state for hsa_step (all device buffers, caller-owned). */
typedef struct {
  float* x;            /* fp32 [N, C] latent, advanced in place */
  float* v_hat;        /* fp32 [N, C] velocity of each token's latest active step */
  float* v_hat_prev;   /* fp32 [N, C] the velocity before that */
  float* v_fresh;      /* fp32 [N, C] this step's head output (rows of A_i written) */
  float* score;        /* fp32 [N] last selector scores */
  uint8_t* g;          /* uint8 [N] group id per token */
  uint8_t* mask;       /* uint8 [N] active mask of the current iteration */
  int32_t* active_idx; /* int32 [N] ascending active tokens (first |A_i| valid) */
  float* h;            /* fp32 [N, D] hidden rows */
  void* const* k_cache;/* host array of L device pointers, bf16 [N, D] each */
  void* const* v_cache;/* host array of L device pointers, bf16 [N, D] each */
} hsa_state;

typedef struct hsa_ctx hsa_ctx;

/*
 * Create a context for one model shape and group layout ([TS] 2.1).
 *   cfg      (host) model shape.
 *   T        total steps.
 *   budgets  (host) s_1..s_K: s_1 == T, strictly decreasing, each divides T.
 *   counts   (host) n_1..n_K tokens per group, sum == N.
 *   K        number of groups, 1..8.
 *   m        phase-aware window ([TS] 2.4): the first m and last m iterations
 *            are full passes for all tokens; 0 disables it; 2m <= T.
 *   stream   cudaStream_t to launch on (NULL = legacy default stream).
 *   out      (host) receives the context.
 * Allocates the context's scratch (compact activations sized for |A| = N,
 * selector histograms, the device error flag) with cudaMalloc.  On failure
 * *out is NULL and nothing is leaked.
 */
hsa_status hsa_create(const hsa_model_cfg* cfg, int T, const int* budgets, const int* counts,
                      int K, int m, void* stream, hsa_ctx** out);

/* Free the context and its scratch.  Synchronises its stream first.  NULL is a no-op. */
void hsa_destroy(hsa_ctx* ctx);

/* Message for the last failing call on ctx (never NULL).  ctx may be NULL for hsa_create errors. */
const char* hsa_last_error(const hsa_ctx* ctx);

/* Replace the stream used by later calls. */
hsa_status hsa_set_stream(hsa_ctx* ctx, void* stream);

/* Synchronise the stream, then read and clear the device error flag. */
hsa_status hsa_sync_check(hsa_ctx* ctx);

/*
 * Failure-detection self-test.  Launches one kernel whose mbarrier wait is
 * never satisfied; the same bounded wait the pipelined kernels use gives up
 * after timeout_us microseconds (1..2000000) and records a timeout in the
 * device flag.  The next hsa_sync_check then returns HSA_ERR_TIMEOUT and
 * clears the flag; the context stays usable.  Nothing faults or hangs.
 */
hsa_status hsa_selftest_timeout(hsa_ctx* ctx, int timeout_us);

/* Number of kernels this context has launched so far (host counter, no sync). */
uint64_t hsa_kernel_launches(const hsa_ctx* ctx);

/*
 * Per-launch timing of the calls above, for measuring the kernels inside a
 * running step (no counterpart on the pages: instrumentation).  While on, every
 * kernel launch of the context is bracketed by two CUDA events on its stream
 * and its algorithmic work is added up per class:
 *   0 attention   (hsa_attention, hsa_attention_kv; work = 4 n n_kv D FLOP)
 *   1 GEMM        (QKV, out-projection, MLP, linear; work = 2 M Ncols K FLOP)
 *   2 row kernels (LN gather, KV scatter, embed, head; work = bytes moved)
 *   3 per-token   (schedule, score, selection, Euler; work = 0)
 * hsa_kernel_times synchronises the stream, writes the first n_classes
 * classes' totals (launch calls, summed event milliseconds, work) to out, and
 * clears them.  Events are taken from a pool the context owns.  Off by
 * default; not meant for use under stream capture.
 */
typedef struct {
  uint64_t calls;
  double ms;
  double work;
} hsa_kernel_class_time;

hsa_status hsa_time_kernels(hsa_ctx* ctx, int on);
hsa_status hsa_kernel_times(hsa_ctx* ctx, hsa_kernel_class_time* out, int n_classes);

/*
 * |A_i| computed on the host from the group counts ([TS] 2.1): the sum of n_k
 * over the groups active at iteration i.  Valid when g holds exactly counts[k]
 * tokens of group k, which the initial split and hsa_select_groups guarantee.
 * Returns -1 if i is outside [0, T).
 */
int hsa_n_active(const hsa_ctx* ctx, int i);

/*
 * Group schedule ([TS] 2.1, 2.4).  Token n is active at iteration i iff
 * i mod (T / s_{g[n]}) == 0, or i is inside the phase window.
 *   g           (device) uint8 [N] group ids, each < K.
 *   mask        (device) uint8 [N] out: 1 if active.
 *   active_idx  (device) int32 [N] out: active tokens in ascending order.
 *   n_active_dev(device) int32 [1] out, may be NULL: |A_i| as counted on the GPU.
 *   n_active    (host)   out, may be NULL: |A_i| from hsa_n_active (no sync).
 * A group id >= K counts as inactive and sets the device check flag.
 */
hsa_status hsa_schedule(hsa_ctx* ctx, int i, const uint8_t* g, uint8_t* mask, int32_t* active_idx,
                        int32_t* n_active_dev, int* n_active);

/*
 * Per-token L1 relative change of the velocity ([TS] 2.1, Dynamic Selection):
 *   score[n] = sum_c |v_cur[n,c] - v_prev[n,c]| / (sum_c |v_prev[n,c]| + 1e-6)
 * in float32, each sum in channel order 0..C-1, one IEEE division.
 *   v_prev, v_cur (device) fp32 [N, C];  score (device) fp32 [N] out.
 */
hsa_status hsa_score(hsa_ctx* ctx, const float* v_prev, const float* v_cur, float* score);

/*
 * Group assignment from a score buffer ([TS] 2.1): tokens ranked by (score
 * descending, index ascending); the first n_1 get group 0 (budget T), the
 * next n_2 group 1, and so on.  Exact and deterministic (integer radix select).
 *   score (device) fp32 [N], finite and >= 0 (a NaN sets the device check flag).
 *   g     (device) uint8 [N] out.
 */
hsa_status hsa_select_from_score(hsa_ctx* ctx, const float* score, uint8_t* g);

/* hsa_score followed by hsa_select_from_score; score may not be NULL. */
hsa_status hsa_select_groups(hsa_ctx* ctx, const float* v_prev, const float* v_cur, float* score,
                             uint8_t* g);

/*
 * Gather + LayerNorm of the active rows (the first stage of the active-only
 * forward, [TS] 2.2 step 1): u[m] = LN(x[idx[m]]) without affine, eps 1e-5.
 *   x   (device) fp32 [N, D];  idx (device) int32 [n];  u (device) bf16 [n, D] out.
 */
hsa_status hsa_ln_gather(hsa_ctx* ctx, const float* x, const int32_t* idx, int n, void* u);

/*
 * QKV projection of the active rows and KV-cache write ([TS] 2.2 steps 1-2):
 * [Q|K|V] = u W_qkv^T; Q goes to the compact buffer q, the fresh K and V rows
 * overwrite rows idx[m] of this layer's caches.
 *   w_qkv (device) bf16 [3D, D];  u (device) bf16 [n, D];  idx (device) int32 [n]
 *   q (device) bf16 [n, D] out;  k_cache, v_cache (device) bf16 [N, D] in/out.
 */
hsa_status hsa_qkv_project(hsa_ctx* ctx, const void* w_qkv, const void* u, const int32_t* idx,
                           int n, void* q, void* k_cache, void* v_cache);

/*
 * The same QKV projection for a sequence-sharded step, with the exchange of
 * the fresh K/V rows folded into the GEMM's epilogue ([TS] 2.2 steps 1-2:
 * every active token's fresh K/V rows must reach every copy of the cache
 * before attention reads it).  Q goes to q as in hsa_qkv_project; every fresh
 * K and V row is stored to row idx[m] of each of the n_caches cache pairs,
 * so that one launch writes this rank's rows into its own cache and, through
 * peer-mapped pointers, into every other rank's copy over NVLink.
 *   w_qkv, u, idx, q as hsa_qkv_project;
 *   k_caches, v_caches (HOST arrays of n_caches pointers, borrowed for the
 *   call): device bf16 [N, D] caches, each on this GPU or a peer GPU's memory
 *   mapped into this process (CUDA IPC or peer access); 1 <= n_caches <= 8.
 * The launch only stores to peer memory (no load reads another GPU).  The
 * caller orders it against the peers' readers: no peer may read the rows
 * before this launch completes (a device-side barrier on the stream after
 * it), and no peer may still be reading a previous step's rows of these
 * caches when it starts.  HSA_ERR_INVALID_ARG for n_caches out of range or a
 * NULL / misaligned pointer; an index outside [0, N) is skipped and reported
 * by hsa_sync_check (HSA_ERR_DEVICE_CHECK).
 */
hsa_status hsa_qkv_project_peers(hsa_ctx* ctx, const void* w_qkv, const void* u,
                                 const int32_t* idx, int n, void* q, void* const* k_caches,
                                 void* const* v_caches, int n_caches);

/*
 * Active-row linear map, the tensor-core building block of the QKV,
 * out-projection and MLP products ([TS] 2.2): out = a w^T, fp32 accumulation.
 *   a (device) bf16 [M, Kd];  w (device) bf16 [Ncols, Kd];  out (device) bf16 [M, Ncols].
 *   Kd % 64 == 0, Ncols % 32 == 0, M >= 0.
 */
hsa_status hsa_linear(hsa_ctx* ctx, const void* a, int M, int Kd, const void* w, int Ncols,
                      void* out);

/*
 * KV-cache write alone ([TS] 2.2 step 2): k_cache[idx[m]] = k_rows[m],
 * v_cache[idx[m]] = v_rows[m].
 *   k_rows, v_rows (device) bf16 [n, D];  k_cache, v_cache (device) bf16 [N, D].
 */
hsa_status hsa_kv_scatter(hsa_ctx* ctx, const void* k_rows, const void* v_rows,
                          const int32_t* idx, int n, void* k_cache, void* v_cache);

/*
 * The same KV-cache write from packed rows, as a sequence-sharded step
 * receives them after gathering every rank's fresh rows ([TS] 2.2 step 2):
 * k_cache[idx[m]] = kv_rows[m][0 .. D), v_cache[idx[m]] = kv_rows[m][D .. 2D).
 *   kv_rows (device) bf16 [n, 2D];  idx (device) int32 [n], each < N;
 *   k_cache, v_cache (device) bf16 [N, D].  An index outside [0, N) is skipped
 *   and reported by hsa_sync_check (HSA_ERR_DEVICE_CHECK).
 */
hsa_status hsa_kv_scatter_packed(hsa_ctx* ctx, const void* kv_rows, const int32_t* idx, int n,
                                 void* k_cache, void* v_cache);

/*
 * Full-context attention of the active queries ([TS] 2.2 steps 3-4):
 * per head, o[m] = softmax(q[m] K^T / sqrt(d)) V over all N cached rows,
 * fp32 accumulation, online softmax.  Cost O(n * N).
 *   q (device) bf16 [n, D];  k_cache, v_cache (device) bf16 [N, D];  o (device) bf16 [n, D] out.
 */
hsa_status hsa_attention(hsa_ctx* ctx, const void* q, int n, const void* k_cache,
                         const void* v_cache, void* o);

/*
 * The same attention against an explicit set of n_kv key/value rows, e.g. the
 * text tokens of cross-attention ([TS] 2.2 step 4 names cross-attention as
 * work that skipped tokens do not incur): o[m] = softmax(q[m] K^T / sqrt(d)) V
 * per head over the n_kv rows.
 *   q (device) bf16 [n, D];  k, v (device) bf16 [n_kv, D];  o (device) bf16 [n, D] out.
 * HSA_ERR_SHAPE if n_kv < 1.
 */
hsa_status hsa_attention_kv(hsa_ctx* ctx, const void* q, int n, const void* k, const void* v,
                            int n_kv, void* o);

/*
 * Out-projection on the active rows, added into the residual rows
 * ([TS] 2.2 step 4): x[idx[m]] += o[m] W_o^T.
 *   w_o (device) bf16 [D, D];  o (device) bf16 [n, D];  x (device) fp32 [N, D] in/out.
 */
hsa_status hsa_out_proj_residual(hsa_ctx* ctx, const void* w_o, const void* o,
                                 const int32_t* idx, int n, float* x);

/*
 * MLP on the active rows ([TS] 2.2 step 4):
 * x[idx[m]] += GELU(LN(x[idx[m]]) W_1^T) W_2^T (exact erf GELU, no biases).
 *   w_1 (device) bf16 [F, D];  w_2 (device) bf16 [D, F];  x (device) fp32 [N, D] in/out.
 * Uses the context's scratch for the LN output and the [n, F] hidden.
 */
hsa_status hsa_mlp_residual(hsa_ctx* ctx, const void* w_1, const void* w_2, float* x,
                            const int32_t* idx, int n);

/*
 * The stages above with the timestep modulation of a conditioned block (the
 * reading of hsa_layer_forward_cond below; [TS] 2.2 step 4 names conditioning
 * only as work skipped tokens do not incur), for callers that run a
 * conditioned block stage by stage, such as a sequence-sharded step:
 *   hsa_ln_gather_mod:            u[m] = LN(x[idx[m]]) * (1 + scale) + shift
 *   hsa_out_proj_residual_gated:  x[idx[m]] += gate * (o[m] W_o^T)
 *   hsa_mlp_residual_mod:         x[idx[m]] += gate * GELU(u2 W_1^T) W_2^T with
 *                                 u2 = LN(x[idx[m]]) * (1 + scale) + shift
 * shift, scale, gate (device) fp32 [D], 16-byte aligned; shift and scale are
 * both given or both NULL (no modulation), gate NULL means 1.  Other
 * arguments, layouts and errors as the unmodulated calls.
 */
hsa_status hsa_ln_gather_mod(hsa_ctx* ctx, const float* x, const int32_t* idx, int n, void* u,
                             const float* shift, const float* scale);
hsa_status hsa_out_proj_residual_gated(hsa_ctx* ctx, const void* w_o, const void* o,
                                       const int32_t* idx, int n, float* x, const float* gate);
hsa_status hsa_mlp_residual_mod(hsa_ctx* ctx, const void* w_1, const void* w_2, float* x,
                                const int32_t* idx, int n, const float* shift,
                                const float* scale, const float* gate);

/*
 * One transformer block on the active set ([TS] 2.2): LN -> QKV (K/V written
 * into the caches) -> attention of the n queries against all N cached rows
 * -> out-projection + residual -> LN -> MLP + residual.  Only rows idx of x
 * and of the caches change.
 *   w (host) weights;  x (device) fp32 [N, D];  idx (device) int32 [n], ascending,
 *   each < N;  k_cache, v_cache (device) bf16 [N, D].
 */
hsa_status hsa_layer_forward(hsa_ctx* ctx, const hsa_layer_weights* w, float* x,
                             const int32_t* idx, int n, void* k_cache, void* v_cache);

/* Text cross-attention of a conditioned block: its weights and the text
 * tokens' keys and values, fixed for the whole sampling run. */
typedef struct {
  const void* w_q;    /* (device) bf16 [D, D] query projection */
  const void* w_o;    /* (device) bf16 [D, D] output projection */
  const void* k_txt;  /* (device) bf16 [n_txt, D] */
  const void* v_txt;  /* (device) bf16 [n_txt, D] */
  int n_txt;          /* >= 1 */
} hsa_cross_attn;

/*
 * A conditioned block on the active set.  The pages name timestep conditioning
 * and text cross-attention only as work skipped tokens do not incur ([TS] 2.2
 * step 4) and give no architecture, so this follows the usual video-DiT form:
 *   u   = LN(x) * (1 + scale_a) + shift_a;  QKV, K/V into the caches, attention
 *         over all N cached rows;  x += gate_a * (o W_o^T)
 *   x  += W_oc Attn(LN(x) W_qc^T, k_txt, v_txt)            (if xa != NULL)
 *   u2  = LN(x) * (1 + scale_m) + shift_m;  x += gate_m * (GELU(u2 W_1^T) W_2^T)
 * with mod (device, fp32 [6, D], 16-byte aligned) holding the rows
 * shift_a, scale_a, gate_a, shift_m, scale_m, gate_m of this iteration.
 * mod == NULL and xa == NULL is hsa_layer_forward.  Only rows idx of x and of
 * the caches change.  Errors as hsa_layer_forward; HSA_ERR_SHAPE if
 * xa->n_txt < 1, HSA_ERR_INVALID_ARG for a NULL or misaligned pointer.
 */
hsa_status hsa_layer_forward_cond(hsa_ctx* ctx, const hsa_layer_weights* w, const float* mod,
                                  const hsa_cross_attn* xa, float* x, const int32_t* idx, int n,
                                  void* k_cache, void* v_cache);

/*
 * Embed the active latent rows: h[idx[m]] = x_lat[idx[m]] W_in^T.
 *   w_in (device) fp32 [D, C];  x_lat (device) fp32 [N, C];  h (device) fp32 [N, D].
 */
hsa_status hsa_embed(hsa_ctx* ctx, const float* w_in, const float* x_lat, const int32_t* idx,
                     int n, float* h);

/*
 * Velocity head on the active rows: v_fresh[idx[m]] = LN(h[idx[m]]) W_head^T.
 *   w_head (device) fp32 [C, D];  h (device) fp32 [N, D];  v_fresh (device) fp32 [N, C].
 */
hsa_status hsa_head(hsa_ctx* ctx, const float* w_head, const float* h, const int32_t* idx,
                    int n, float* v_fresh);

/*
 * Cached Euler update over all N tokens in one pass ([TS] 2.3):
 *   v_hat_prev[n] = mask[n] ? v_hat[n]   : v_hat_prev[n]
 *   v_hat[n]      = mask[n] ? v_fresh[n] : v_hat[n]
 *   x[n]          = x[n] + (sigma_next - sigma_i) * v_hat[n]
 * in float32 with one rounding per operation (no fused multiply-add).
 *   x, v_hat, v_hat_prev (device) fp32 [N, C] in/out;  v_fresh (device) fp32 [N, C];
 *   mask (device) uint8 [N].
 */
hsa_status hsa_euler_step(hsa_ctx* ctx, float* x, float* v_hat, float* v_hat_prev,
                          const float* v_fresh, const uint8_t* mask, float sigma_i,
                          float sigma_next);

/*
 * The same cached Euler update, and in the same pass the score of the
 * re-grouping that follows it ([TS] 2.1, Dynamic Selection; [TS] 2.3): after
 * the update above,
 *   score[n] = sum_c |v_hat[n,c] - v_hat_prev[n,c]| / (sum_c |v_hat_prev[n,c]| + 1e-6)
 * in float32, sums in channel order, bit for bit what hsa_score writes for
 * (v_hat_prev, v_hat).  A re-grouping step thus reads the velocity caches
 * once; hsa_select_from_score then assigns the groups.
 *   score (device) fp32 [N] out; the other arguments as hsa_euler_step.
 *   A NaN, negative or infinite score is reported by hsa_sync_check
 *   (HSA_ERR_DEVICE_CHECK).
 */
hsa_status hsa_euler_step_score(hsa_ctx* ctx, float* x, float* v_hat, float* v_hat_prev,
                                const float* v_fresh, const uint8_t* mask, float sigma_i,
                                float sigma_next, float* score);

/*
 * One global iteration i of the HSA loop ([TS] 2.1-2.3): schedule -> embed
 * the active latent rows -> every layer on A_i -> head -> cached Euler over
 * all N -> (when ``regroup`` is non-zero and T/s_K <= i < T-1) re-select the
 * groups from v_hat_prev and v_hat (the Euler pass writes the scores, as
 * hsa_euler_step_score).  No host synchronisation.
 *   w (host) model weights;  s (host) state;  sigma_i, sigma_next the noise
 *   levels of iterations i and i+1.
 */
hsa_status hsa_step(hsa_ctx* ctx, const hsa_model_weights* w, const hsa_state* s, int i,
                    float sigma_i, float sigma_next, int regroup);

/*
 * Conditioning of one iteration for hsa_step_cond: per layer, the modulation
 * vectors of this iteration (they follow the timestep, so the caller passes
 * new ones each iteration) and the text cross-attention (fixed for the run).
 * See hsa_layer_forward_cond for what they do; the pages give no
 * architecture for either ([TS] 2.2 step 4 only says skipped tokens incur no
 * cross-attention).
 */
typedef struct {
  const float* const* mod;  /* host array of L device pointers, fp32 [6, D] each (a NULL
                               entry: that layer unmodulated), or NULL for none */
  const hsa_cross_attn* xa; /* host array of L entries, or NULL for no cross-attention */
} hsa_cond;

/*
 * hsa_step with conditioned blocks: every layer runs hsa_layer_forward_cond
 * with cond->mod[l] and cond->xa[l].  cond == NULL is hsa_step.  Arrays are
 * read during the call only.  Errors as hsa_step and hsa_layer_forward_cond.
 */
hsa_status hsa_step_cond(hsa_ctx* ctx, const hsa_model_weights* w, const hsa_state* s,
                         const hsa_cond* cond, int i, float sigma_i, float sigma_next,
                         int regroup);

/*
 * Group selection without any device allocation.  The paper has no
 * counterpart: this is a service for callers that cannot call cudaMalloc,
 * such as a host framework that owns all device memory through its own pool
 * and forbids a library to allocate, or a latency-critical serving loop
 * where cudaMalloc's implicit device synchronisation would stall other work.
 *
 * Same result as hsa_select_groups (scores, then exact group assignment with
 * ties broken by token index), but it needs no context: the scores and cut
 * keys live in one static device array of the library, sized for at most
 * HSA_SELECT_STATIC_MAX_N tokens (512 KiB of scores + 64 B of cut keys +
 * 256 B for the error flag), which every GPU that loads the library holds
 * until the process exits.
 *   v_prev, v_cur (device) fp32 [N, 16];  counts (host) n_1..n_K, sum == N;
 *   g (device) uint8 [N] out;  stream cudaStream_t (NULL = legacy default).
 * Returns HSA_ERR_SCRATCH_LIMIT when N > HSA_SELECT_STATIC_MAX_N, and the
 * other argument errors of hsa_create / hsa_select_groups; there is no
 * message string.  Calls no cudaMalloc or cudaFree.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call before any stream capture.  The
 * address belongs to the device's primary context: after cudaDeviceReset the
 * next call finds a new context and looks the address up again (make that
 * call, too, outside stream capture).
 * All calls share the array and it keeps the last call's contents; calls
 * that overlap on the GPU race on it.  Device-side checks (a NaN score) are
 * not reported by this call.
 */
#define HSA_SELECT_STATIC_MAX_N 131072
hsa_status hsa_select_groups_static(const float* v_prev, const float* v_cur, int N,
                                    const int* counts, int K, uint8_t* g, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HSA_H_ */

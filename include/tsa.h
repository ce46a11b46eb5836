/*
 * tsa.h -- C ABI of the Token Sparse Attention prefill hot path (sm_100a).
 *
 * The operation is the per-layer prefill attention of Token Sparse Attention:
 * every KV head scores all L tokens, keeps its own top-K subset, compresses
 * Q/K/V to that subset, runs causal attention on the compressed tensors and
 * scatters the result back to length L (zeros at dropped rows), ready for the
 * caller's residual add.
 *
 * Sources (page title, then the section / figure):
 *   [P1] "Token Sparse Attention Long Context" (skillsdirectory skill page):
 *        Step 1 TokenScorer.score_tokens ("entropy") and select_top_k;
 *        Step 2 gather_tokens and scatter_attention_output;
 *        Step 3 SparseAttentionHead.forward.
 *   [P2] "Token Sparse Attention: Efficient Long-Context Inference with
 *        Interleaved Token Selection" (sciencestack): Figure 3 (Stage 1
 *        compresses Q, K, V per head to a token subset; Stage 2 attends on the
 *        compressed tensors and scatters back to the full sequence layout
 *        before the residual add); TL;DR (head-specific subsets).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Layout, row-major and contiguous ("BHLD"):
 *     q   [B, Hq,  L, D]     k, v [B, Hkv, L, D]     out [B, Hq, L, D]
 *     scores [B, Hkv, L] float32      perm [B, Hkv, L] int32
 *   dtype of q/k/v/out: TSA_F32 (float) or TSA_BF16 (bfloat16).
 *   Query head h belongs to KV group g = h / G, G = Hq / Hkv.
 * - Every tensor pointer is DEVICE memory owned by the caller, 16-byte aligned.
 *   The library allocates nothing, frees nothing and does not synchronise in
 *   the compute calls: work is enqueued on `stream` (a cudaStream_t passed as
 *   void*, NULL = legacy default stream) and the call returns.  The documented
 *   exceptions are tsa_forward_host (host buffers, copies on the stream) and
 *   tsa_forward_coverage (one synchronisation to bring the chosen budgets back).
 * - `budget_host` is a HOST array of B*Hkv int32 kept-token counts, one per
 *   (batch, KV head), read during the call (grid planning needs it).  A budget
 *   <= 0 is TSA_ERR_INVALID_ARG; a budget > L is clamped to L, as [P1] Step 3
 *   clamps k to the sequence length.
 * - `ws` is a device workspace of at least tsa_workspace_size() bytes, owned by
 *   the caller, zero-filled once before first use (tsa_workspace_init).  It
 *   holds a device status word; calls sharing one workspace must be ordered on
 *   one stream.
 * - Argument errors are returned synchronously and nothing is launched.
 *   Device-side errors (a bounded wait that ran out, a failed bounds check)
 *   are recorded in the workspace status word and reported by
 *   tsa_check_status().
 * - Supported: D in {64, 128}; Hq % Hkv == 0; G = Hq/Hkv in {1,2,4,8,16};
 *   1 <= window <= L; G*window <= 256; B*Hq*L < 2^31; B*Hkv <= 1024.
 *   bf16 runs on tcgen05 tensor-core kernels, f32 on exact SIMT kernels.
 *   There is no CPU path.
 */
#ifndef TSA_H_
#define TSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TSA_API __attribute__((visibility("default")))
#else
#define TSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tsa_status {
  TSA_OK = 0,
  TSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or budget   */
  TSA_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shapes/dtypes */
  TSA_ERR_WORKSPACE = 3,     /* workspace smaller than tsa_workspace_size()   */
  TSA_ERR_CUDA = 4,          /* a CUDA runtime call failed                    */
  TSA_ERR_TIMEOUT = 5,       /* a device-side bounded wait ran out            */
  TSA_ERR_DEVICE_BOUNDS = 6  /* a device-side index check failed              */
} tsa_status;

typedef enum tsa_dtype { TSA_F32 = 0, TSA_BF16 = 1 } tsa_dtype;

/* Problem shape.  scale <= 0 selects 1/sqrt(D), the 1/sqrt(head dim) of
 * [P1] Step 1 and Step 3. */
typedef struct tsa_desc {
  int32_t B, Hq, Hkv, L, D;
  int32_t dtype; /* tsa_dtype */
  float scale;
} tsa_desc;

/* Bytes of device workspace needed by any call on this shape and window. */
TSA_API size_t tsa_workspace_size(const tsa_desc* desc, int32_t window);

/* Zero the workspace header (status word, counters).  Enqueued on `stream`. */
TSA_API tsa_status tsa_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * tsa_score -- per-KV-head token importance ([P1] Step 1, "entropy":
 * softmax of q.k/sqrt(d) over keys, summed over queries).
 * For each query head h and each of the last `window` query positions
 * p in [L-window, L): logits_j = scale * q[p].k[j] over keys j <= p, softmax
 * over j, accumulated into scores[b, h/G, j] (summed over the window queries
 * and over the G query heads of the KV group).  Each KV head's scores sum to
 * window*G.  Output: scores [B,Hkv,L] float32, fully overwritten.
 */
TSA_API tsa_status tsa_score(const tsa_desc* desc, const void* q, const void* k, int32_t window,
                     float* scores, void* ws, size_t ws_bytes, void* stream);

/*
 * tsa_select -- top-K per KV head ([P1] Step 1 select_top_k; [P2] Figure 3
 * per-head subsets; budgets may differ per head).  For (b,g) with
 * K = min(budget_host[b*Hkv+g], L): keeps the K largest scores, ties broken
 * toward the lower index, +0.0 == -0.0.  perm[b,g,0:K] lists the kept token
 * indices ascending, perm[b,g,K:L] the dropped ones ascending.  Scores must
 * be finite.  Bit-exact and deterministic.
 */
TSA_API tsa_status tsa_select(const tsa_desc* desc, const float* scores, const int32_t* budget_host,
                      int32_t* perm, void* ws, size_t ws_bytes, void* stream);

/*
 * tsa_attend -- gather, causal attention on the compressed tensors, scatter
 * ([P1] Steps 2-3; [P2] Figure 3 Stages 1-2).  For query head h, group g,
 * K = min(budget, L), kept row i < K at original position p_i = perm[b,g,i]:
 *   out[b,h,p_i] = sum_{r <= i} softmax_r(scale * q[b,h,p_i].k[b,g,p_r]) v[b,g,p_r]
 * (causal by original positions; perm[b,g,0:K] must be strictly ascending).
 * Every dropped position perm[b,g,K:L] gets +0 in all D columns.  `out` is
 * fully overwritten.  perm must be a permutation of [0,L) per (b,g) in the
 * layout tsa_select produces; indices outside [0,L) are a device bounds error.
 */
TSA_API tsa_status tsa_attend(const tsa_desc* desc, const void* q, const void* k, const void* v,
                      const int32_t* perm, const int32_t* budget_host, void* out, void* ws,
                      size_t ws_bytes, void* stream);

/*
 * tsa_out_proj -- the attention output's projection added to the residual
 * ("Token Sparse Attention Long Context" skill page, Step 3: out_proj applied
 * to the attention output of the selected tokens, then scattered back to full
 * length; [P2] Figure 3: the residual connection is added after the scatter):
 *   x[b, p, :] += sum over query heads h whose KV group g = h / G kept p of
 *                 attn_out[b, h, p, :] . w_o[:, h*D : (h+1)*D]^T
 * for every position p kept by at least one group; rows no group kept are
 * left untouched.  The projection is bias-free (the multi-head form of the
 * page's out_proj on the concatenated head outputs).
 *   attn_out: device [B, Hq, L, D] in desc->dtype, the layout tsa_attend
 *             writes; rows at positions a head's group dropped are not read.
 *   perm, budget_host: the selection tsa_select produced (same rules as
 *             tsa_attend).
 *   w_o:      device [hidden, Hq*D] row-major in desc->dtype (an nn.Linear
 *             weight, out_features x in_features).
 *   x:        device [B, L, hidden] in desc->dtype, holding the residual on
 *             entry; read and written in place (fp32 accumulation, one
 *             rounding to the dtype per element).
 *   ws:       device workspace of tsa_out_proj_workspace_size() bytes, 16-byte
 *             aligned, status word first (tsa_check_status reads it).
 * Supported: Hkv <= 16 per batch entry; hidden a multiple of 256 for bf16
 * (tcgen05 kernel), of 64 for f32 (SIMT kernel).  One memset and five kernel
 * launches on `stream`; returns after enqueueing.  TSA_ERR_INVALID_ARG for a
 * bad pointer, budget or hidden; TSA_ERR_UNSUPPORTED outside the shapes;
 * TSA_ERR_WORKSPACE for a short workspace.
 */
TSA_API size_t tsa_out_proj_workspace_size(const tsa_desc* desc);
TSA_API tsa_status tsa_out_proj(const tsa_desc* desc, const void* attn_out, const int32_t* perm,
                                const int32_t* budget_host, const void* w_o, int32_t hidden, void* x, void* ws,
                                size_t ws_bytes, void* stream);

/*
 * tsa_zero_dropped -- the zero rows of the scatter on their own ([P1] Step 2
 * scatter_attention_output builds the full-length output from zeros; [P2]
 * Figure 3 scatters into the full sequence layout): for each (b, g) with
 * K = min(budget_host[b*Hkv+g], L), out[b, h, p, :] = +0 for every dropped
 * position p in perm[b,g,K:L] and every query head h of group g.  Kept rows
 * are not touched.  tsa_attend writes these zeros itself; this call is the
 * same step as one standalone kernel (for callers that write the kept rows
 * another way, and to measure the step).  Same pointer, budget and
 * permutation rules as tsa_attend.
 */
TSA_API tsa_status tsa_zero_dropped(const tsa_desc* desc, const int32_t* perm, const int32_t* budget_host,
                                    void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * tsa_score_noalloc -- tsa_score without a caller workspace, for callers that
 * cannot allocate device memory (for example a plugin inside an engine that
 * owns all device memory, or a latency-critical loop that must not call
 * cudaMalloc).  The pages have no counterpart: this is a deployment variant.
 * Same arguments, layout, kernels and result as tsa_score (tensor-core passes
 * for bf16, SIMT passes for f32); the per-split partials go to a fixed 1 MiB
 * array built into the library, reserved on every GPU that loads it until the
 * process exits.  Checks run in this order: the shape (as tsa_score), then
 * the partials' size -- B*Hkv * splits * rows * 8 bytes above 1 MiB returns
 * TSA_ERR_WORKSPACE, with splits = min(ceil(L/128), 18) and rows = 128 or 256
 * (G*window <= 128 or not) in bf16, splits = min(ceil(L/64), 74) and rows =
 * G*window rounded up to 64 in f32; the 32/8-head, window-64 layer fits at
 * B = 1 up to L = 131072 in bf16 (295 KB) and up to B = 64 at L <= 128 --
 * then the pointers (TSA_ERR_INVALID_ARG).  The first call made
 * with a device current looks up the array's device address; make that first
 * call before any stream capture.  All calls share the array: calls whose
 * kernels overlap on the GPU race and give wrong scores, so order them on one
 * stream.  Device-side errors go to a status word of the library, read (and
 * cleared) by tsa_check_status(NULL, 0, stream).  Allocates nothing.
 */
TSA_API tsa_status tsa_score_noalloc(const tsa_desc* desc, const void* q, const void* k, int32_t window,
                                     float* scores, void* stream);

/*
 * tsa_attend_block_sparse -- tsa_attend composed with block-sparse attention
 * inside the compressed space ("Token Sparse Attention: Efficient Long-Context
 * Inference with Interleaved Token Selection", Figures 1 and 5b: the method on
 * top of a block-sparse attention kernel).  block_mask: device uint8
 * [B*Hkv][nb][nb], nb = ceil(L / 128), row-major; entry (i, j) of KV group
 * (b, g) enables the block of compacted query rows [128 i, 128 i + 128) of its
 * G query heads against compacted keys [128 j, 128 j + 128); the causal mask
 * still applies inside.  Disabled key tiles are skipped (no loads, no MMAs)
 * when every query row of a CTA has them disabled.  A kept row that sees no
 * key outputs zeros; dropped rows are zeros as in tsa_attend.  Same other
 * arguments and rules as tsa_attend.
 */
TSA_API tsa_status tsa_attend_block_sparse(const tsa_desc* desc, const void* q, const void* k, const void* v,
                                           const int32_t* perm, const int32_t* budget_host,
                                           const uint8_t* block_mask, void* out, void* ws, size_t ws_bytes,
                                           void* stream);

/*
 * tsa_select_coverage -- tsa_select with each (b, g) budget chosen from a
 * token coverage tau in [0, 1] ("Token Sparse Attention: Efficient
 * Long-Context Inference with Interleaved Token Selection": dynamic token
 * coverage; Figures 1 and 5).  Each score s has the integer mass
 * floor(clamp(s, 0, 256) * 2^S), S = 55 - ceil(log2 L) (NaN counts as 0);
 * with M the head's total and T = M - floor(double(M) * tau), K is the
 * smallest k >= 1 whose k top-ranked tokens (tsa_select's order) carry mass
 * >= T (K = 1 when T = 0).  perm is written as by tsa_select with that K, and
 * budget_dev_out (device int32[B*Hkv], 4-byte aligned) receives the K values.
 * One kernel launch; returns after enqueueing.  TSA_ERR_INVALID_ARG for tau
 * outside [0, 1] or NaN and the pointer rules of tsa_select.
 */
TSA_API tsa_status tsa_select_coverage(const tsa_desc* desc, const float* scores, double tau, int32_t* perm,
                                       int32_t* budget_dev_out, void* ws, size_t ws_bytes, void* stream);

/*
 * tsa_attend_accumulate -- tsa_attend, but scatter-ADD into an existing output
 * ([P1] Step 2 scatter_add_attention_output, `full_output[b, indices] +=
 * attention_output`): out[b,h,p_i] += attention row i for the kept rows, in
 * fp32 then rounded once to the output dtype; dropped rows keep their value.
 * Same arguments and rules as tsa_attend; `out` is read and written.
 */
TSA_API tsa_status tsa_attend_accumulate(const tsa_desc* desc, const void* q, const void* k, const void* v,
                                         const int32_t* perm, const int32_t* budget_host, void* out, void* ws,
                                         size_t ws_bytes, void* stream);

/*
 * tsa_forward -- tsa_score, tsa_select and tsa_attend in sequence on `stream`.
 * scores_or_null / perm_or_null: where to keep the intermediates; NULL puts
 * them in the workspace.
 */
TSA_API tsa_status tsa_forward(const tsa_desc* desc, const void* q, const void* k, const void* v,
                       int32_t window, const int32_t* budget_host, float* scores_or_null,
                       int32_t* perm_or_null, void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * tsa_forward_coverage -- tsa_score, tsa_select_coverage and tsa_attend in
 * sequence, budgets chosen from the coverage tau.  The attention grid is
 * sized from the budgets, so the call copies them into budget_host_out (host
 * int32[B*Hkv]) and SYNCHRONISES `stream` between the selection and the
 * attention; it returns after enqueueing the attention.  Same buffers and
 * workspace rule as tsa_forward.
 */
TSA_API tsa_status tsa_forward_coverage(const tsa_desc* desc, const void* q, const void* k, const void* v,
                                        int32_t window, double tau, int32_t* budget_host_out,
                                        float* scores_or_null, int32_t* perm_or_null, void* out, void* ws,
                                        size_t ws_bytes, void* stream);

/*
 * tsa_forward_host -- tsa_forward on HOST inputs and output, all on `stream`;
 * out_dev is copied back to out_host in full.  The inputs reach the caller's
 * device buffers q_dev/k_dev/v_dev in one of two ways:
 * - q_host and v_host both mapped into the device's address space (pinned
 *   with the mapped flag; cudaHostAlloc memory is mapped under unified
 *   addressing): only what the step reads crosses the host link ([P1] Step 2
 *   gathers only the selected tokens; [P2] Figure 3, Stage 1).  K is copied
 *   in full (every key is scored), and the last `window` rows of every query
 *   head are copied.  After the selection a kernel reads the kept rows of Q
 *   (the G heads of each KV group) and of V in place and writes them to the
 *   same positions of q_dev / v_dev.  Other rows of q_dev / v_dev are not
 *   written.
 * - otherwise: one cudaMemcpyAsync of each whole input, then tsa_forward.
 * The result in out_host is the same either way.  The call returns after
 * enqueueing; the host buffers must stay valid until the stream reaches that
 * point.  TSA_ERR_DEVICE_BOUNDS (status word) for a permutation entry
 * outside [0, L).
 */
TSA_API tsa_status tsa_forward_host(const tsa_desc* desc, const void* q_host, const void* k_host,
                            const void* v_host, int32_t window, const int32_t* budget_host,
                            void* out_host, void* q_dev, void* k_dev, void* v_dev, void* out_dev,
                            void* ws, size_t ws_bytes, void* stream);
/* Host-to-device bytes tsa_forward_host moves for these arguments: K in full,
 * plus either the window rows of Q and the kept rows of Q (G per kept
 * position) and of V (mapped q_host and v_host), or all of Q and V.  0 for an
 * invalid shape, window or budget. */
TSA_API size_t tsa_forward_host_h2d_bytes(const tsa_desc* desc, int32_t window, const int32_t* budget_host,
                                          const void* q_host, const void* v_host);

/*
 * tsa_drift -- representation drift between two hidden-state tensors
 * ("Token Sparse Attention Long Context" skill page, Step 4,
 * LayerStabilityAnalyzer.compute_representation_drift):
 *     drift = 1 - mean_r < a_r / max(|a_r|, 1e-12), b_r / max(|b_r|, 1e-12) >
 * over the `rows` rows of h_before (a) and h_after (b), each [rows, hidden]
 * row-major in `dtype` (TSA_F32 or TSA_BF16), device memory, 16-byte aligned,
 * with hidden * sizeof(element) a multiple of 16 bytes.  Rows are accumulated
 * in fp32, the mean in fp64.
 *   row_cos_or_null: device float[rows] receiving each row's cosine, or NULL.
 *   drift:           device double[1] receiving the drift (8-byte aligned).
 *   ws:              device workspace of at least tsa_drift_workspace_size()
 *                    bytes, 16-byte aligned, owned by the caller; calls on
 *                    one workspace must be ordered on one stream.
 * One memset and one kernel launch on `stream`; the call returns after
 * enqueueing.  TSA_ERR_INVALID_ARG for rows < 1, a bad dtype, hidden, pointer
 * or alignment; TSA_ERR_WORKSPACE for a short workspace.
 */
TSA_API size_t tsa_drift_workspace_size(void);
TSA_API tsa_status tsa_drift(int64_t rows, int32_t hidden, int32_t dtype, const void* h_before,
                             const void* h_after, float* row_cos_or_null, double* drift, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * tsa_layer_stable -- the same page's LayerStabilityAnalyzer.is_layer_stable
 * window rule on host data: *stable = 1 when history (n drifts, newest last,
 * host memory) holds at least `window` entries and the mean of the newest
 * `window` is strictly below `threshold`, else 0.  TSA_ERR_INVALID_ARG for
 * window < 1, n < 0, a NULL `stable`, or a NULL history with n > 0.
 */
TSA_API tsa_status tsa_layer_stable(const double* history, int32_t n, int32_t window, double threshold,
                                    int32_t* stable);

/* Synchronise `stream`, return the device status recorded in `ws` (TSA_OK,
 * TSA_ERR_TIMEOUT or TSA_ERR_DEVICE_BOUNDS) and clear it.  ws = NULL reads
 * the status word of tsa_score_noalloc on the current device instead. */
TSA_API tsa_status tsa_check_status(void* ws, size_t ws_bytes, void* stream);

/* Static description of a status code. */
TSA_API const char* tsa_status_string(tsa_status s);

/*
 * Failure-detection and accounting hooks (testing; no counterpart on the pages).
 * tsa_debug_set_wait_limit: poll budget of every device-side bounded wait of
 *   later launches in this process (0 restores the default of about a second).
 * tsa_debug_wait_never_set: launch one block that waits on a workspace flag
 *   nothing sets; with a small limit it records TSA_ERR_TIMEOUT and returns.
 */
TSA_API void tsa_debug_set_wait_limit(uint64_t polls);
/* Number of kernels this library has launched in this process (all devices). */
TSA_API uint64_t tsa_debug_launch_count(void);
/* Number of those that were the two-SM attention kernel (d = 128 on CTA pairs,
 * cta_group::2), which tsa_attend, tsa_attend_accumulate,
 * tsa_attend_block_sparse and the forward calls use in place of the one-SM
 * kernel while the environment variable TSA_ATTEND_CTA_PAIRS is set to a
 * value other than "0" (read at every launch; same arguments and results
 * within the attention tolerance; off by default). */
TSA_API uint64_t tsa_debug_cta_pair_launch_count(void);
TSA_API tsa_status tsa_debug_wait_never_set(void* ws, size_t ws_bytes, void* stream);
/* y = 2^x through the FMA-pipe exponential the scoring kernel uses for one
 * pair of values in three (device arrays of n floats, n even, 16-byte aligned). */
TSA_API tsa_status tsa_debug_exp2(const float* x, float* y, int32_t n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TSA_H_ */

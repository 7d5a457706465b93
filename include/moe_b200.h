/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) sparse MoE FFN layer forward.
 *
 * The layer, in order (page tags as in the library's design notes):
 *   route      router GEMM -> softmax/sigmoid affinity -> choice-only bias ->
 *              group-limited pre-selection -> top-k -> renormalised gate weights
 *   permute    per-expert counts -> capacity / token-order drop -> offsets ->
 *              expert-contiguous rows (stable in token order) -> row gather
 *   grouped_ffn SwiGLU expert FFN over variable-size row groups (also the
 *              always-on shared experts, as one group over all tokens)
 *   combine    gate-weighted sum of each token's expert rows (+ shared output)
 *   router_stats / bias_update  f_i, P_i, aux, z-loss, CV, dead, drops; the
 *              aux-loss-free sign update of the selection bias.
 *
 * Conventions shared by every entry point
 *   - Return value: a moe_status_t (0 = MOE_OK).  Arguments are checked on the
 *     host before anything is enqueued; an invalid call enqueues nothing.
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless the
 *     comment says "host".  The library never allocates or frees device memory
 *     and keeps no pointer after a call returns.
 *   - All work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream).  No call synchronises the host.
 *   - Device pointers must be 16-byte aligned; tensors are dense row-major.
 *   - Kernel-side failures that the host cannot see (a bounded wait that ran
 *     out) are recorded in a device status word; read it with
 *     moe_device_status() after synchronising.
 *   - Integer outputs are deterministic: the same inputs give the same bytes on
 *     every run.  Floating-point outputs are deterministic too (no atomics on
 *     any floating-point accumulation).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* bad size, null pointer, misalignment, k > N ... */
  MOE_ERR_UNSUPPORTED = 2,        /* valid request outside what the kernels implement */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3,
  MOE_ERR_CUDA = 4,               /* a CUDA runtime call failed (launch, tensor map) */
  MOE_ERR_DEVICE_TIMEOUT = 5      /* a device-side bounded wait gave up */
} moe_status_t;

enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 };
enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 };
enum {
  MOE_CAP_DROPLESS = 0,           /* no capacity limit */
  MOE_CAP_CEIL_CF_T_OVER_N = 1,   /* C = ceil((cf*T)/N)  (default capacity reading) */
  MOE_CAP_CF_K_T_OVER_N_FLOOR = 2 /* C = max(floor(cf*k*T/N), k)  (the Practice page's code) */
};

/* Shape and routing options of one MoE layer.  Plain data, host memory. */
typedef struct moe_config {
  int64_t T;                 /* tokens (batch x sequence, flattened), >= 0          */
  int32_t d_model;           /* d, multiple of 8                                    */
  int32_t n_experts;         /* N routed experts, 1..512                            */
  int32_t top_k;             /* k, 1..min(N, 16)                                    */
  int32_t d_ff;              /* f, routed expert hidden size, multiple of 8         */
  int32_t score_fn;          /* MOE_SCORE_*                                         */
  int32_t renorm;            /* 1: w = s_sel / sum s_sel; 0: w = s_sel              */
  int32_t n_groups;          /* <= 1: no group limit; else divides N, <= 32         */
  int32_t topk_groups;       /* groups kept per token (group limit on)              */
  int32_t group_score_topn;  /* group score = sum of its topn best scores, >= 1     */
  int32_t capacity_mode;     /* MOE_CAP_*                                           */
  int32_t x_dtype;           /* MOE_DTYPE_*: x, expert weights, h, y all this type  */
  int32_t shared_sink;       /* 1: one shared expert joins the weight normalisation:
                                w_gate has N+1 rows, row N scoring the shared expert */
  double capacity_factor;    /* cf (> 0) for the capacity modes                     */
} moe_config_t;

/* Router statistics, written by moe_router_stats (device memory). */
typedef struct moe_stats {
  float aux;                 /* alpha * N * sum_e f_e P_e                            */
  float aux_raw;             /* N * sum_e f_e P_e (1 under uniform routing)          */
  float z;                   /* mean_t (logsumexp_e z[t,e])^2                        */
  float z_loss;              /* z_coef * z                                           */
  float cv;                  /* population std / mean of pre-capacity counts        */
  float cv_kept;             /* same over kept (post-capacity) counts               */
  float bias_norm;           /* ||b||_2 (0 when no bias)                             */
  int32_t dead;              /* experts with zero selections                        */
  int32_t dropped_slots;     /* k*T - R                                             */
  int32_t dropped_tokens;    /* tokens whose k slots were all dropped               */
  int32_t R;                 /* kept rows                                           */
  int32_t near_ties;         /* tokens whose selection margin (moe_route's margin) is
                                below the near-tie threshold; -1 when not counted   */
  int64_t T;                 /* tokens covered (summed over ranks after a reduction) */
  int32_t reserved[2];
} moe_stats_t;

/* Length, in doubles, of the sufficient-statistics vector of moe_router_stats_partial. */
#define MOE_STATS_PARTIAL_LEN(n_experts) (3 * (n_experts) + 5)

/* ---------------------------------------------------------------------------
 * Sizing queries (host only; no device work).
 * ------------------------------------------------------------------------- */

/* Per-expert capacity C for cfg (host out).  Dropless gives C = INT64_MAX.
 * Capacity: "容量因子与专家并行（工程视角）" on the llm-compass MoE page
 * (capacity = cf * tokens / N) and "容量因子、token dropping 与一笔算不清的隐形税" on the
 * Practice page (C = cf * k * T / N; its code floors and keeps at least k). */
int moe_capacity(const moe_config_t* cfg, int64_t* capacity);

/* Rows of the p_partial buffer written by moe_route (host out). */
int moe_route_partials(const moe_config_t* cfg, int32_t* nblk);

/* Bytes of scratch `ws` needed by moe_route and moe_permute for cfg (host out):
 * the larger of the two, so one buffer serves both when the calls are ordered on
 * one stream.  Calls that share a workspace must not overlap on the GPU. */
int moe_workspace_size(const moe_config_t* cfg, size_t* bytes);

/* ---------------------------------------------------------------------------
 * moe_route -- fused router GEMM + affinity + bias + group limit + top-k + renorm.
 *
 * Defines: "路由的数学形式：softmax、top-k 与那些必须做的小动作" (Practice page:
 * logits -> softmax -> top-k -> renormalise; the router has no bias term), the
 * llm-compass page's "稀疏门控与 Top-k 路由" (g = softmax(TopK(xW_g))) and its
 * "负载均衡：从 aux loss 到 aux-loss-free" (selection on s_i + b_i, weights from s_i).
 *
 *   x            [T, d]   cfg->x_dtype (fp32 or bf16)
 *   w_gate       [N, d]   fp32 router weight (kept in fp32; never quantised), or NULL
 *                on the tensor-core path (bf16 x, N <= 256) when `ws` holds the split
 *                written by moe_route_prepare for this cfg and weight (`ws` must then
 *                not be shared with moe_permute)
 *   logit_offset [N] fp32 or NULL: added to every token's logits
 *   bias         [N] fp32 or NULL: added to the affinity for selection only
 *   topk_idx     [T, k] int32 out: experts in descending selection score;
 *                equal scores -> lower expert index first
 *   topk_w       [T, k] fp32 out: gate weights (raw affinity, renormalised)
 *   lse          [T] fp32 out: logsumexp of the logits (z-loss input)
 *   p_partial    [nblk, N] fp32 out: per-block sums over tokens of the
 *                normalised affinity (softmax probs, or s / sum s for sigmoid);
 *                nblk from moe_route_partials
 *   margin       [T] fp32 out or NULL: selection score of the k-th pick minus the
 *                best eligible expert left out, min'ed with the last-kept minus
 *                best-dropped group score (+inf when nothing is left out)
 *   shared_w     [T] fp32 out (only with cfg->shared_sink, else NULL): weight of the
 *                shared expert's output.  With the sink, w_gate has N+1 rows; the
 *                affinity covers all N+1 logits (softmax over N+1, or sigmoids), top-k
 *                chooses among the N routed experts, and the k routed weights and the
 *                shared weight are normalised together (MoE common-taste page, section
 *                11, shared-expert sink); lse covers the N+1 logits; p_partial uses
 *                the routed affinities normalised over the routed experts.
 *   ws           scratch of at least moe_workspace_size() bytes (clobbered)
 * The router GEMM is fp32-equivalent: fp32 FMA, or for bf16 x and N <= 256 the
 * tensor cores over an exact three-way bf16 split of w_gate (every product exact,
 * fp32 accumulation).  T = 0 is a no-op.
 * ------------------------------------------------------------------------- */
int moe_route(const moe_config_t* cfg, const void* x, const float* w_gate,
              const float* logit_offset, const float* bias,
              int32_t* topk_idx, float* topk_w, float* lse, float* p_partial,
              float* margin, float* shared_w, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_route_prepare -- the router weight's exact three-way bf16 split, once per weight.
 *
 * The tensor-core router (bf16 x, N <= 256; see moe_route) multiplies x by the
 * split W_g = W_hi + W_mid + W_lo (each piece the next 8 significant bits, so every
 * product is exact).  moe_route computes the split on every call; a caller whose
 * router weight changes less often than it routes writes it once here and then
 * calls moe_route with w_gate = NULL and ws = this buffer.  No page defines this
 * call: it is the reuse of a pure function of the weight.
 *   w_gate    [N, d] fp32 (N + 1 rows with cfg->shared_sink)
 *   prepared  device out, at least moe_route_prepare_size() bytes, 16-byte aligned
 * Errors: MOE_ERR_UNSUPPORTED off the tensor-core path; MOE_ERR_WORKSPACE_TOO_SMALL.
 * ------------------------------------------------------------------------- */
int moe_route_prepare_size(const moe_config_t* cfg, size_t* bytes);
int moe_route_prepare(const moe_config_t* cfg, const float* w_gate, void* prepared, size_t bytes,
                      void* stream);

/* ---------------------------------------------------------------------------
 * moe_permute -- counts, capacity drop in token order, offsets, row maps, gather.
 *
 * Defines: Practice page "容量因子、token dropping" (per-expert hard cap; the
 * earliest occupants are kept, reproducibly) and "专家并行与 all-to-all" (stable
 * grouping by destination so one grouped GEMM covers all experts); dropped slots
 * contribute zero.
 *
 *   x            [T, d] x_dtype
 *   topk_idx     [T, k] int32, each row k distinct experts in [0, N); a slot whose
 *                id is outside [0, N) or repeats an earlier slot of its token is
 *                treated as dropped (row -1) and recorded as MOE_ERR_INVALID_ARG
 *                in the device status word (see moe_device_status)
 *   counts       [N] int32 out: selections per expert before capacity (c_e)
 *   offsets      [N+1] int32 out: exclusive scan of kept_e = min(c_e, C)
 *   row_of_slot  [T, k] int32 out: row of slot (t, j) in x_perm, -1 if dropped
 *   token_of_row [T*k] int32 out: token of each row (entries >= R untouched)
 *   x_perm       [T*k, d] x_dtype out: x_perm[row] = x[token_of_row[row]]
 *                (rows >= R untouched); rows of expert e are its kept slots in
 *                ascending token order.  NULL skips the gather (x may then be
 *                NULL too), e.g. when moe_permute_fp8 fills FP8 rows instead
 *   n_dropped    [2] int32 out: {dropped slots, tokens with all k slots dropped}
 *   ws           scratch of at least moe_workspace_size() bytes (contents on
 *                entry ignored; clobbered)
 * ------------------------------------------------------------------------- */
int moe_permute(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                int32_t* counts, int32_t* offsets, int32_t* row_of_slot,
                int32_t* token_of_row, void* x_perm, int32_t* n_dropped,
                void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_grouped_ffn -- SwiGLU FFN over G variable-size row groups in one pass.
 *
 * Defines: "专家并行与 all-to-all" on the Practice page (expert-contiguous rows let
 * one grouped GEMM compute every expert) and the llm-compass "MoE 层结构" (each
 * expert is an FFN).  The pages name three matrices per expert without spelling
 * SwiGLU out; the form used is y = W2 (silu(W1 x) * (W3 x)), silu(z) = z/(1+e^-z).
 *
 *   x_rows   [rows_cap, d] x_dtype: rows offsets[g] .. offsets[g+1]-1 belong to
 *            group g; rows_cap >= offsets[G]
 *   offsets  [G+1] int32 (device), non-decreasing, offsets[0] = 0
 *   w1, w3   [G, f, d] x_dtype (gate and up projections)
 *   w2       [G, d, f] x_dtype (down projection)
 *   h_scratch[rows_cap, f] x_dtype: the SwiGLU hidden rows (written, then read)
 *   y_rows   [rows_cap, d] x_dtype out (rows >= offsets[G] untouched)
 * bf16: tcgen05 tensor cores, fp32 accumulation, h rounded to bf16.
 * fp32: fp32 FMA throughout.  Shared experts: G = 1, offsets = {0, T},
 * x_rows = x, f = n_shared * d_ff_shared with the experts' matrices concatenated
 * along f.
 * ------------------------------------------------------------------------- */
int moe_grouped_ffn(const moe_config_t* cfg, const void* x_rows, int64_t rows_cap,
                    const int32_t* offsets, int32_t G,
                    const void* w1, const void* w3, const void* w2, int32_t f,
                    void* h_scratch, void* y_rows, void* stream);

/* ---------------------------------------------------------------------------
 * moe_grouped_ffn_shared -- moe_grouped_ffn with the shared expert in the same launches.
 *
 * The shared expert (the Practice page's and the llm-compass "MoE 层结构" always-on
 * expert) is the same SwiGLU FFN applied to every token: here it is one more group,
 * of all T tokens with its own weights, scheduled with the routed groups inside the
 * two grouped-GEMM launches (one tile list, no second pair of launches, no launch
 * tails between them).  Same arithmetic as moe_grouped_ffn on each part: the routed
 * outputs equal moe_grouped_ffn's and the shared outputs equal moe_grouped_ffn with
 * G = 1, offsets = {0, T}, bit for bit.
 *   x_rows, rows_cap, offsets, G, w1, w3, w2, f  the routed groups, as for
 *                     moe_grouped_ffn
 *   h_scratch         [rows_cap + T, f] bf16 (written, then read): the groups' hidden
 *                     rows, then the shared expert's (row rows_cap + t for token t)
 *   y_rows            [rows_cap + T, d] bf16 out: the groups' rows (rows >= offsets[G]
 *                     and < rows_cap untouched), then the shared expert's output for
 *                     token t at row rows_cap + t
 *   x                 [T, d] bf16: the shared expert's input (token order)
 *   ws1, ws3          [f, d] bf16; ws2 [d, f] bf16: the shared expert, hidden width f
 *                     (the routed experts' f; shared experts of another total width
 *                     take moe_grouped_ffn with G = 1)
 * Errors: MOE_ERR_UNSUPPORTED unless bf16, or when rows_cap + T exceeds INT32_MAX;
 * MOE_ERR_INVALID_ARG as for moe_grouped_ffn, for G > 511, T < 0, or a NULL or
 * misaligned buffer.  T = 0 is moe_grouped_ffn.
 * ------------------------------------------------------------------------- */
int moe_grouped_ffn_shared(const moe_config_t* cfg, const void* x_rows, int64_t rows_cap,
                           const int32_t* offsets, int32_t G, const void* w1, const void* w3, const void* w2,
                           int32_t f, void* h_scratch, void* y_rows, const void* x, int64_t T, const void* ws1,
                           const void* ws3, const void* ws2, void* stream);

/* ---------------------------------------------------------------------------
 * moe_grouped_ffn_gate_up, moe_grouped_ffn_down -- the two passes of moe_grouped_ffn
 * as separate calls (bf16), so a caller can run the shared expert's first pass on
 * another stream while the router and the permutation run, and its second pass in
 * the routed second pass's launch.  Same kernels and arithmetic as moe_grouped_ffn
 * and moe_grouped_ffn_shared: bit-identical results.
 *
 * moe_grouped_ffn_gate_up: h_rows[r] = silu(x_rows[r] W1[g]^T) * (x_rows[r] W3[g]^T)
 *   for the rows r of each group g.  x_rows [rows_cap, d], w1/w3 [G, f, d], h_rows
 *   [rows_cap, f] (bf16); offsets [G+1] (device).  G <= 512.
 * moe_grouped_ffn_down: y_rows[r] = h_rows[r] W2[g]^T for the groups' rows; with T > 0
 *   and ws2 [d, f] also y_rows[rows_cap + t] = h_rows[rows_cap + t] ws2^T for t < T (the
 *   shared expert's rows, whose first pass the caller ran), in the same launch.  h_rows
 *   [rows_cap + T, f], y_rows [rows_cap + T, d].  G <= 511.
 * Errors: MOE_ERR_UNSUPPORTED unless cfg->x_dtype is bf16, or when the rows exceed
 * INT32_MAX; MOE_ERR_INVALID_ARG for a bad G, f, rows_cap or T, for T > 0 without ws2
 * (or ws2 with T = 0), or a NULL or misaligned buffer.  No rows is a no-op.
 * ------------------------------------------------------------------------- */
int moe_grouped_ffn_gate_up(const moe_config_t* cfg, const void* x_rows, int64_t rows_cap, const int32_t* offsets,
                            int32_t G, const void* w1, const void* w3, int32_t f, void* h_rows, void* stream);
int moe_grouped_ffn_down(const moe_config_t* cfg, const void* h_rows, int64_t rows_cap, const int32_t* offsets,
                         int32_t G, const void* w2, int32_t f, void* y_rows, int64_t T, const void* ws2,
                         void* stream);

/* ---------------------------------------------------------------------------
 * moe_grouped_ffn_gather -- moe_grouped_ffn reading each row straight from x.
 *
 * The same grouped SwiGLU FFN (same sources, same arithmetic, bit-identical
 * output) with row r's input x[token_of_row[r]] fetched by the first GEMM itself,
 * so the expert-ordered copy of x (moe_permute's x_perm) is never written: call
 * moe_permute with x_perm = NULL and pass its token_of_row here.  The first GEMM's
 * producer warp copies the rows with cp.async, 16 bytes per lane, into the same
 * swizzled tiles a TMA box would give.  This trades time for memory: T k d fewer
 * elements held, but on the DeepSeek-V3-shaped layer (T = 16384, d = 7168, 256
 * experts, k = 8, shared expert fused) the grouped FFN took 14.9 ms against 11.6 ms
 * over the copy, which itself takes 0.4 ms.  With ws1, ws3, ws2 given, the shared expert
 * over all T tokens rides in the same two launches as one more group, as in
 * moe_grouped_ffn_shared (its rows read from x in order).
 *   x             [T, d] bf16 (device), the tokens in token order
 *   token_of_row  [rows_cap] int32 (device): token of each row; read for rows
 *                 < offsets[G] only.  An entry outside [0, T) is replaced by token
 *                 0 and recorded as MOE_ERR_INVALID_ARG in the device status word
 *   offsets, w1, w3, w2, f, rows_cap: as for moe_grouped_ffn
 *   h_scratch, y_rows  [rows_cap (+ T with the shared expert), f] and [.., d] bf16:
 *                 the routed rows, then the shared expert's T rows
 *   ws1, ws3 [f, d], ws2 [d, f] bf16, or all three NULL: the shared expert, of the
 *                 routed width f
 * Errors: MOE_ERR_UNSUPPORTED unless cfg->x_dtype is bf16 and d % 64 == 0 (the
 * rows are moved in whole 64-column steps), or when rows_cap (+ T) exceeds
 * INT32_MAX; MOE_ERR_INVALID_ARG as for moe_grouped_ffn, or for G > 511, T < 0, a
 * NULL token_of_row, or only some of ws1, ws3, ws2.  T = 0, or rows_cap = 0 without
 * the shared expert, is a no-op.
 * ------------------------------------------------------------------------- */
int moe_grouped_ffn_gather(const moe_config_t* cfg, const void* x, int64_t T, const int32_t* token_of_row,
                           int64_t rows_cap, const int32_t* offsets, int32_t G, const void* w1, const void* w3,
                           const void* w2, int32_t f, void* h_scratch, void* y_rows, const void* ws1,
                           const void* ws3, const void* ws2, void* stream);

/* ---------------------------------------------------------------------------
 * FP8 expert compute with fine-grained block scaling.
 *
 * Defines: the MoE common-taste page, section 2 (its table lists FP8 / MXFP8 expert
 * compute as a strong candidate), and the Practice page "精度怎么定" (matmuls in
 * FP8 with fine-grained precision assignment, the router kept at higher
 * precision).  The pages give no scheme; the reading used is the DeepSeek-V3 one:
 * E4M3 codes (OCP FP8, bias 7, max 448, no infinities), one fp32 scale per 1 x 128
 * block of activations and per 128 x 128 block of weights, scale = amax / 448
 * (1 for an all-zero block), code = E4M3(x / scale) rounded to nearest even with
 * saturation, x / scale in fp32.  The router (moe_route) is unchanged.
 * ------------------------------------------------------------------------- */

/* moe_quantize_fp8 -- block-quantise a bf16 matrix.
 *   x          [rows, cols] bf16 (device), cols % 128 == 0
 *   block_rows 1 (activations: 1 x 128 blocks) or 128 (weights: 128 x 128 blocks)
 *   q          [rows, cols] uint8 E4M3 codes out
 *   scales     [ceil(rows / block_rows), cols / 128] fp32 out
 * Stacked expert weights [G, f, d] are passed as rows = G * f; with f % 128 == 0
 * no block spans two experts.  Errors: MOE_ERR_INVALID_ARG for a bad shape, a
 * NULL or misaligned pointer (x, q 16-byte; scales 4-byte). */
int moe_quantize_fp8(const void* x, int64_t rows, int32_t cols, int32_t block_rows, uint8_t* q,
                     float* scales, void* stream);

/* moe_permute_fp8 -- quantise x (1 x 128 blocks) and scatter it into expert rows.
 * Each token's row is read and quantised once; its codes and scales are written
 * to every row the permutation gave it (row_of_slot from moe_permute, which may
 * be called with x_perm = NULL to skip its own bf16 gather) and, when xq is not
 * NULL, to row t of token-order buffers (the shared experts' input).
 *   x           [T, d] bf16, d % 128 == 0
 *   row_of_slot [T, k] int32 or NULL (token-order output only)
 *   xq_perm     [rows, d] uint8 out, xs_perm [rows, d / 128] fp32 out
 *   xq, xs      [T, d] uint8 and [T, d / 128] fp32 out, or NULL
 * Errors: MOE_ERR_UNSUPPORTED unless x is bf16 with d % 128 == 0;
 * MOE_ERR_INVALID_ARG for NULL or misaligned buffers. */
int moe_permute_fp8(const moe_config_t* cfg, const void* x, const int32_t* row_of_slot, uint8_t* xq_perm,
                    float* xs_perm, uint8_t* xq, float* xs, void* stream);

/* moe_grouped_ffn_fp8 -- the grouped SwiGLU FFN of moe_grouped_ffn on E4M3 codes.
 *   xq_rows, xs_rows  [rows_cap, d] codes, [rows_cap, d / 128] scales
 *   offsets           [G+1] int32 (device), as for moe_grouped_ffn
 *   w1q/w1s, w3q/w3s  [G f, d] codes, [G f / 128, d / 128] scales
 *   w2q/w2s           [G d, f] codes, [G d / 128, f / 128] scales
 *   hq/hs_scratch     [rows_cap, f] codes, [rows_cap, f / 128] scales (written, read)
 *   y_rows            [rows_cap, d] bf16 out (rows >= offsets[G] untouched)
 * Tensor cores (E4M3 x E4M3, fp32 accumulation) over one 128-wide K block at a
 * time; the two block scales are applied in fp32 as each block is accumulated.
 * h = silu(W1 x) * (W3 x) is computed in fp32 and re-quantised in 1 x 128 blocks.
 * Errors: MOE_ERR_UNSUPPORTED unless bf16 config with d % 128 == f % 128 == 0;
 * MOE_ERR_INVALID_ARG for G outside [1, 512], NULL or misaligned buffers. */
int moe_grouped_ffn_fp8(const moe_config_t* cfg, const uint8_t* xq_rows, const float* xs_rows,
                        int64_t rows_cap, const int32_t* offsets, int32_t G, const uint8_t* w1q,
                        const float* w1s, const uint8_t* w3q, const float* w3s, const uint8_t* w2q,
                        const float* w2s, int32_t f, uint8_t* hq_scratch, float* hs_scratch, void* y_rows,
                        void* stream);

/* ---------------------------------------------------------------------------
 * MXFP8 expert compute (OCP Microscaling FP8).
 *
 * Defines: the MoE common-taste page, section 2 (its table names MXFP8 expert
 * compute).  Format: E4M3 codes; every 32 consecutive elements along a row (the
 * contraction dimension of the GEMM operand) share one E8M0 scale byte b, value
 * 2^(b - 127), with b - 127 = floor(log2 amax) - 8 clamped to [-127, 127]
 * (b = 0 for an all-zero block); code = E4M3(x / 2^(b - 127)), round to nearest
 * even, saturating at 448.  The tensor cores apply the scales inside the MMA
 * (block-scaled MMA).
 *
 * Scale layout ("tile atoms", the order the GEMM consumes them in): the rows of
 * an operand are cut into tiles of 128 -- for rows grouped by expert (offsets),
 * tile i of group g starts at row offsets[g] + 128 i and the tiles are numbered
 * in group order; a plain matrix is one group.  The scales of tile t and 128-wide
 * K block kb fill the 512-byte atom at byte (t * (cols / 128) + kb) * 512; row m
 * of the tile, scale j of the K block (elements 128 kb + 32 j .. + 31) is at byte
 * 16 (m mod 32) + 4 floor(m / 32) + j of the atom.  A buffer for `rows` rows in G
 * groups needs (ceil(rows / 128) + G) * (cols / 128) * 512 bytes (plain matrix:
 * ceil(rows / 128) * (cols / 128) * 512); bytes of rows past a group's end are
 * unspecified.
 * ------------------------------------------------------------------------- */

/* moe_quantize_mxfp8 -- quantise a bf16 matrix along its rows.
 *   x   [rows, cols] bf16 (device, 16-byte aligned), cols % 128 == 0
 *   q   [rows, cols] uint8 E4M3 codes out (8-byte aligned)
 *   sf  E8M0 scales out, tile atoms of the plain matrix (layout above)
 * Expert weights [G, f, d] are quantised as rows = G * f (blocks never span rows).
 * Errors: MOE_ERR_INVALID_ARG for a bad shape or a NULL or misaligned pointer. */
int moe_quantize_mxfp8(const void* x, int64_t rows, int32_t cols, uint8_t* q, uint8_t* sf, void* stream);

/* moe_permute_mxfp8 -- moe_permute_fp8 with MXFP8 rows: each token's row is read
 * and quantised once and written (codes and scales) to every kept row given by
 * row_of_slot and, when q is not NULL, to row t of token-order buffers.
 *   x            [T, d] bf16, d % 128 == 0
 *   topk_idx     [T, k] int32 (the experts of the slots)
 *   row_of_slot  [T, k] int32 from moe_permute, or NULL (token order only)
 *   offsets      [N+1] int32 from moe_permute (the groups of the tile-atom layout)
 *   q_perm       [T*k, d] codes out; sf_perm: scales out, tile atoms grouped by offsets
 *   q, sf        [T, d] codes and plain-matrix tile atoms out, or NULL
 * Errors: MOE_ERR_UNSUPPORTED unless bf16 with d % 128 == 0 and N <= 1024;
 * MOE_ERR_INVALID_ARG for NULL or misaligned buffers. */
int moe_permute_mxfp8(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, const int32_t* row_of_slot,
                      const int32_t* offsets, uint8_t* q_perm, uint8_t* sf_perm, uint8_t* q, uint8_t* sf,
                      void* stream);

/* moe_grouped_ffn_mxfp8 -- the grouped SwiGLU FFN of moe_grouped_ffn on MXFP8 operands.
 *   xq_rows, xsf_rows  [rows_cap, d] codes; scales as tile atoms grouped by offsets
 *   offsets            [G+1] int32 (device), as for moe_grouped_ffn
 *   w1q/w1sf, w3q/w3sf [G f, d] codes; scales as plain-matrix tile atoms
 *   w2q/w2sf           [G d, f] codes; scales as plain-matrix tile atoms
 *   hq/hsf_scratch     [rows_cap, f] codes; scales as tile atoms grouped by offsets
 *                      (written by the first pass, read by the second)
 *   y_rows             [rows_cap, d] bf16 out (rows >= offsets[G] untouched)
 * One fp32 TMEM accumulator over the whole K range (block-scaled tcgen05 MMA);
 * h = silu(W1 x) * (W3 x) in fp32, re-quantised to MXFP8 along f.
 * Errors: MOE_ERR_UNSUPPORTED unless a bf16 config with d % 128 == f % 128 == 0;
 * MOE_ERR_INVALID_ARG for G outside [1, 512], NULL or misaligned (16-byte) buffers. */
int moe_grouped_ffn_mxfp8(const moe_config_t* cfg, const uint8_t* xq_rows, const uint8_t* xsf_rows,
                          int64_t rows_cap, const int32_t* offsets, int32_t G, const uint8_t* w1q,
                          const uint8_t* w1sf, const uint8_t* w3q, const uint8_t* w3sf, const uint8_t* w2q,
                          const uint8_t* w2sf, int32_t f, uint8_t* hq_scratch, uint8_t* hsf_scratch,
                          void* y_rows, void* stream);

/* ---------------------------------------------------------------------------
 * NVFP4 expert compute.
 *
 * Defines: the MoE common-taste page, section 2 (its table names NVFP4 beside FP8 /
 * MXFP8 expert compute, without the scheme).  Reading (NVIDIA's two-level NVFP4):
 * E2M1 codes (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), one unsigned E4M3 scale b per
 * 16 consecutive elements of a row (the GEMM's contraction dimension) and one fp32
 * scale g per tensor.  In fp32, in this order: b = E4M3(amax_16 / fp32(6 g)) (round
 * to nearest even, saturating at 448), s = fp32(b g), code = E2M1(fp32(x / s)) (round
 * to nearest even, saturating at 6); b = 0 gives zero codes.  Weights take
 * g = amax / (6 * 448) per expert matrix; activations (x rows, h) take g = 1.
 * Codes are packed two per byte, element 2i in the low nibble: a [rows, cols] matrix
 * takes rows * cols / 2 bytes.  Scales are stored as tile atoms: rows cut into tiles
 * of 128 (per group for grouped rows: tile i of group g starts at offsets[g] + 128 i,
 * tiles numbered in group order); the 512-byte atom of tile t and 64-wide K chunk c
 * sits at (t * (cols / 64) + c) * 512 and holds scale j (elements 64 c + 16 j ..
 * 64 c + 16 j + 15) of the tile's row m at byte 16 (m % 32) + 4 (m / 32) + j.  A
 * buffer for R rows in G groups takes (ceil(R / 128) + G) * (cols / 64) * 512 bytes.
 * The tensor cores apply the E4M3 block scales inside the MMA
 * (tcgen05.mma.kind::mxf4nvf4.block_scale.scale_vec::4X); the epilogue multiplies by
 * the weights' tensor scales.
 * ------------------------------------------------------------------------- */

/* moe_quantize_nvfp4 -- quantise a bf16 matrix along its rows.
 *   x            [rows, cols] bf16 (device, 16-byte aligned), cols % 64 == 0
 *   tensor_rows  0: tensor scale 1 (activations); else rows per tensor (rows %
 *                tensor_rows == 0), each tensor's g = amax / (6 * 448) written to g
 *   q            [rows, cols / 2] uint8 out (4-byte aligned); sf tile atoms out
 *   g            [rows / tensor_rows] fp32 out (unused when tensor_rows == 0)
 * Errors: MOE_ERR_INVALID_ARG for a bad shape or a NULL or misaligned pointer. */
int moe_quantize_nvfp4(const void* x, int64_t rows, int32_t cols, int32_t tensor_rows, uint8_t* q, uint8_t* sf,
                       float* g, void* stream);

/* moe_permute_nvfp4 -- moe_permute_mxfp8 with NVFP4 rows (tensor scale 1): each
 * token's row is read and quantised once and written to every kept row it has
 * (row_of_slot from moe_permute, called with x_perm = NULL), and, when q is not
 * NULL, to row t of token-order buffers (the shared experts' input).
 *   q_perm [rows, d / 2], sf_perm tile atoms of the grouped rows (groups: offsets)
 *   q [T, d / 2], sf tile atoms of the T token rows (one group)
 * Errors: MOE_ERR_UNSUPPORTED unless bf16 with d % 256 == 0 and N <= 1024;
 * MOE_ERR_INVALID_ARG for missing or misaligned buffers. */
int moe_permute_nvfp4(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, const int32_t* row_of_slot,
                      const int32_t* offsets, uint8_t* q_perm, uint8_t* sf_perm, uint8_t* q, uint8_t* sf,
                      void* stream);

/* moe_grouped_ffn_nvfp4 -- the grouped SwiGLU FFN of moe_grouped_ffn on NVFP4 operands.
 *   xq_rows, xsf_rows  [rows_cap, d / 2] codes, grouped tile atoms (tensor scale 1)
 *   offsets            [G+1] int32 (device), as for moe_grouped_ffn
 *   w1q/w1sf/g1, w3q/w3sf/g3  [G f, d / 2] codes, atoms, [G] tensor scales
 *   w2q/w2sf/g2        [G d, f / 2] codes, atoms, [G] tensor scales
 *   hq/hsf_scratch     [rows_cap, f / 2] codes and grouped atoms of h (written, read)
 *   y_rows             [rows_cap, d] bf16 out (rows >= offsets[G] untouched)
 * Tensor cores (E2M1 x E2M1, fp32 accumulation, E4M3 scales applied per 16 elements
 * inside the MMA); h = silu(g1 W1 x) * (g3 W3 x) in fp32, re-quantised with tensor
 * scale 1; y = g2 (W2 h).
 * Errors: MOE_ERR_UNSUPPORTED unless bf16 with d % 256 == 0 and f % 256 == 0;
 * MOE_ERR_INVALID_ARG for G outside [1, 512] or NULL or misaligned buffers. */
int moe_grouped_ffn_nvfp4(const moe_config_t* cfg, const uint8_t* xq_rows, const uint8_t* xsf_rows,
                          int64_t rows_cap, const int32_t* offsets, int32_t G, const uint8_t* w1q,
                          const uint8_t* w1sf, const float* g1, const uint8_t* w3q, const uint8_t* w3sf,
                          const float* g3, const uint8_t* w2q, const uint8_t* w2sf, const float* g2, int32_t f,
                          uint8_t* hq_scratch, uint8_t* hsf_scratch, void* y_rows, void* stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism: the data path around the all-to-all exchange.
 *
 * Defines: the Practice page, "专家并行与 all-to-all": experts are sharded over W
 * ranks (rank of expert e = e / (N / W), N % W == 0); the ranks exchange their
 * per-expert counts before the all-to-all, send each kept (token, expert) row to
 * the rank holding its expert, compute there, and send the results back for the
 * weighted combine.  After moe_permute a rank's rows are ordered by expert, hence
 * by destination rank, so they are the dispatch send buffer as they stand.  The
 * exchange itself (count all-gather, two all-to-alls) is the caller's (NCCL).
 * ------------------------------------------------------------------------- */

/* moe_ep_plan -- split sizes and regroup map of one rank.
 *   offsets_all   [W, N+1] int32 (device): every rank's expert offsets from
 *                 moe_permute (the all-gather of offsets); rank s keeps
 *                 offsets_all[s, e+1] - offsets_all[s, e] rows of expert e
 *   send_splits   [W] int32 out: rows this rank sends to each rank
 *   recv_splits   [W] int32 out: rows this rank receives from each rank
 *   local_offsets [N/W + 1] int32 out: exclusive scan, over this rank's experts, of
 *                 the rows all ranks send it (the groups of the local grouped FFN)
 *   regroup_map   [recv_cap] int32 out: received row q (source-rank major, then
 *                 expert, then row) -> its local row (expert major, then source
 *                 rank, then row); entries past the received total are untouched
 * Errors: MOE_ERR_INVALID_ARG for W < 1, rank outside [0, W), N % W != 0, NULL. */
int moe_ep_plan(const int32_t* offsets_all, int32_t world, int32_t rank, int32_t n_experts, int32_t* send_splits,
                int32_t* recv_splits, int32_t* local_offsets, int32_t* regroup_map, int64_t recv_cap, void* stream);

/* moe_rows_move -- move rows through an index map (no counterpart on the pages:
 * the regroup step of the exchange above).
 *   src, dst   row-major buffers of row_bytes per row (row_bytes % 16 == 0, 16-byte aligned)
 *   map        [rows_cap] int32 (device)
 *   n_rows     device int32 scalar: rows to move (min with rows_cap), or NULL for rows_cap
 *   scatter    0: dst[r] = src[map[r]];  1: dst[map[r]] = src[r]
 * Errors: MOE_ERR_INVALID_ARG for a bad size, flag, NULL or misaligned buffer. */
int moe_rows_move(const void* src, int64_t row_bytes, const int32_t* map, const int32_t* n_rows, int64_t rows_cap,
                  int32_t scatter, void* dst, void* stream);

/* ---------------------------------------------------------------------------
 * The exchange over NVLink peer memory (the Practice page, "专家并行与 all-to-all":
 * dispatch to the expert's rank, compute, send back for the weighted combine; its
 * "通信优化按什么顺序做" asks for the dispatch to be fused with the work around it).
 * Every rank maps every other rank's receive buffer (moe_peer_export on the owner,
 * moe_peer_import elsewhere, handles passed by the caller's all-gather).  A rank's
 * kernels store its rows straight into the owning ranks' receive buffers and read
 * the results back from there; no kernel waits for another rank.  The caller
 * separates the phases with a stream-ordered barrier (any collective on the stream):
 *   moe_ep_peer_plan -> moe_ep_peer_dispatch -> barrier -> local grouped FFN on the
 *   receive buffer (local_offsets from moe_ep_plan) -> barrier ->
 *   moe_combine_peer (one round) or moe_ep_peer_collect + moe_combine (rounds)
 * and, before a receive buffer takes new rows, a barrier after its last readers.
 * A receive buffer is in local-expert order (local expert major, then source rank,
 * then row): the rows moe_ep_plan's regroup map would produce, without the regroup.
 * ------------------------------------------------------------------------- */
#define MOE_PEER_HANDLE_BYTES 72

/* moe_peer_export -- handle of a device buffer for other processes of the node.
 *   ptr      device pointer into a cudaMalloc allocation (e.g. from a caching allocator)
 *   handle   [MOE_PEER_HANDLE_BYTES] host out: the allocation's CUDA IPC handle (64
 *            bytes), then ptr's byte offset inside the allocation (int64)
 * The buffer stays owned by the caller and must outlive every import of it.
 * Errors: MOE_ERR_INVALID_ARG for NULL or a pointer outside any device allocation;
 * MOE_ERR_CUDA when the allocation cannot be shared (e.g. virtual-memory mapped). */
int moe_peer_export(const void* ptr, void* handle);

/* moe_peer_import -- map another process's exported buffer into this one.
 *   handle   [MOE_PEER_HANDLE_BYTES] host: from moe_peer_export in the owner process
 *   ptr      host out: device pointer to the buffer, valid on the calling thread's
 *            current device (peer access over NVLink) until moe_peer_close
 * Importing the same handle again returns the same pointer and counts one more use.
 * Errors: MOE_ERR_INVALID_ARG for NULL or a negative offset; MOE_ERR_CUDA when the
 * runtime cannot open the handle (e.g. the owner process is this process). */
int moe_peer_import(const void* handle, void** ptr);

/* moe_peer_close -- release one import; the mapping goes when its last use does.
 * Errors: MOE_ERR_INVALID_ARG for a pointer that moe_peer_import did not return. */
int moe_peer_close(void* ptr);

/* moe_ep_peer_plan -- where each of this rank's rows lands in one round.
 *   offsets_round [W, N+1] int32 (device): every rank's expert offsets counting only
 *                 the pieces (source, expert) of this round (a piece is wholly in one
 *                 round); the same array moe_ep_plan takes
 *   offsets_own   [N+1] int32 (device): this rank's full offsets from moe_permute
 *   peer_rows     [W] uint64 (device): address of row 0 of each rank's receive buffer
 *                 as this rank sees it (its own buffer at [rank])
 *   row_bytes     bytes per row (d * element size, % 16 == 0); recv_cap rows per buffer
 *   row_addr      [rows, >= offsets_own[N]] uint64 out: row i's address in the receive
 *                 buffer of rank e / (N / W), e its expert; 0 for rows outside the round.
 *                 A row of the round that would land past recv_cap gets 0 and records
 *                 MOE_ERR_INVALID_ARG in the device status word.
 * Errors: MOE_ERR_INVALID_ARG for W < 1, rank outside [0, W), N % W != 0, a bad
 * row_bytes or recv_cap, NULL. */
int moe_ep_peer_plan(const int32_t* offsets_round, const int32_t* offsets_own, int32_t world, int32_t rank,
                     int32_t n_experts, const uint64_t* peer_rows, int64_t row_bytes, int64_t recv_cap,
                     uint64_t* row_addr, void* stream);

/* moe_ep_peer_dispatch -- *row_addr[row_of_slot[t, j]] = x[t] for every slot whose row
 * is not -1 and whose address is not 0: the permutation's row gather and the
 * dispatch in one pass, x read once per token (call moe_permute with x_perm = NULL).
 * The stores are made visible to the whole system before the kernel ends.
 *   x [T, d] cfg->x_dtype (16-byte aligned); row_of_slot [T, k] from moe_permute;
 *   row_addr [rows_cap] from moe_ep_peer_plan.  A row at or past rows_cap moves
 *   nothing and records MOE_ERR_INVALID_ARG in the device status word.
 * Errors: MOE_ERR_INVALID_ARG for a bad config, rows_cap < 0, NULL or misaligned x. */
int moe_ep_peer_dispatch(const moe_config_t* cfg, const void* x, const int32_t* row_of_slot,
                         const uint64_t* row_addr, int64_t rows_cap, void* stream);

/* moe_ep_peer_collect -- y_perm[i] = *row_addr[i] for i < min(*n_rows, rows_cap) with
 * row_addr[i] != 0: one round's results back into this rank's expert-ordered rows.
 *   row_addr [rows_cap] uint64 (device) from moe_ep_peer_plan
 *   n_rows   device int32 scalar: this rank's rows (offsets[N] from moe_permute)
 *   y_perm   [rows_cap, d] cfg->x_dtype out (16-byte aligned)
 * Errors: MOE_ERR_INVALID_ARG for a bad config, rows_cap < 0, NULL row_addr or n_rows,
 * NULL or misaligned y_perm. */
int moe_ep_peer_collect(const moe_config_t* cfg, const uint64_t* row_addr, const int32_t* n_rows, int64_t rows_cap,
                        void* y_perm, void* stream);

/* moe_combine_peer -- moe_combine with the result of row r read at row_addr[r] (a
 * peer's receive buffer) instead of y_perm[r]; a row whose address is 0 counts as
 * dropped.  Same slot order and fp32 accumulation as moe_combine, so the output is
 * bit-identical to moe_combine over the collected rows.
 * Errors: as moe_combine. */
int moe_combine_peer(const moe_config_t* cfg, const uint64_t* row_addr, const int32_t* row_of_slot,
                     const float* topk_w, const void* shared_out, const float* shared_w, void* y, void* stream);

/* ---------------------------------------------------------------------------
 * moe_combine -- y[t] = shared[t] + sum_{j: row >= 0} w[t,j] * y_perm[row(t,j)].
 *
 * Defines: llm-compass "稀疏门控与 Top-k 路由" (y = sum_i g_i E_i(x)) and the Practice
 * page's "共享专家" (the always-on output is added).  Slots in ascending j,
 * fp32 accumulation, no atomics.
 *   y_perm      [R, d] x_dtype; row_of_slot [T, k]; topk_w [T, k] fp32
 *   shared_out  [T, d] x_dtype or NULL; y [T, d] x_dtype out (may alias shared_out)
 *   shared_w    [T] fp32 or NULL: per-token weight of shared_out (NULL: weight 1;
 *               moe_route's shared_w output with the shared-expert sink)
 * ------------------------------------------------------------------------- */
int moe_combine(const moe_config_t* cfg, const void* y_perm, const int32_t* row_of_slot,
                const float* topk_w, const void* shared_out, const float* shared_w, void* y,
                void* stream);

/* ---------------------------------------------------------------------------
 * moe_router_stats -- router statistics in fixed reduction order.
 *
 * Defines: llm-compass "负载均衡" (L_aux = alpha N sum f_i P_i), the Practice page's
 * "负载均衡损失" (equals 1 unscaled under uniform routing) and "MoE 的可观测性"
 * (专家间的尺度漂移 section: drop ratio and per-expert load as the minimum metrics); the landscape page's monitoring list
 * (token drop, usage CV, dead experts, bias norm).  z-loss has no formula on the
 * pages; mean_t (logsumexp_e z)^2 is used.
 *   counts [N], offsets [N+1], p_partial [nblk, N], lse [T], n_dropped [2],
 *   bias [N] or NULL  (all from the calls above)
 *   margin [T] fp32 or NULL (moe_route's margin): tokens with margin < near_tie are
 *          counted in stats->near_ties (-1 when margin is NULL)
 *   stats  moe_stats_t out; f_out [N], p_out [N] fp32 out (either may be NULL)
 * ------------------------------------------------------------------------- */
int moe_router_stats(const moe_config_t* cfg, const int32_t* counts, const int32_t* offsets,
                     const float* p_partial, const float* lse, const int32_t* n_dropped,
                     const float* margin, float near_tie, const float* bias, float alpha,
                     float z_coef, moe_stats_t* stats, float* f_out, float* p_out, void* stream);

/* ---------------------------------------------------------------------------
 * Global statistics over data-parallel ranks: moe_router_stats_partial on every
 * rank -> element-wise sum of the vectors over ranks (the caller's all-reduce) ->
 * moe_router_stats_finalize.  The result equals moe_router_stats on the
 * concatenated batch (the landscape page's TL;DR and 实践要点: balance statistics
 * should be global, not per micro-batch; the Practice page's load-balance section
 * on the batch the statistics are taken over).
 *
 * moe_router_stats_partial: arguments as moe_router_stats; partial
 *   [MOE_STATS_PARTIAL_LEN(N)] fp64 out: c_e, kept_e, sum_t s-hat_te for every
 *   expert, then sum_t lse_t^2, T, dropped slots, dropped tokens, near-ties.
 * moe_router_stats_finalize: partial as above (summed over ranks); stats, f_out,
 *   p_out as in moe_router_stats; counts_out [N] int32 out or NULL: the summed
 *   c_e (input of moe_bias_update, so every rank applies the same update).
 * ------------------------------------------------------------------------- */
int moe_router_stats_partial(const moe_config_t* cfg, const int32_t* counts, const int32_t* offsets,
                             const float* p_partial, const float* lse, const int32_t* n_dropped,
                             const float* margin, float near_tie, double* partial, void* stream);
int moe_router_stats_finalize(const moe_config_t* cfg, const double* partial, const float* bias,
                              float alpha, float z_coef, moe_stats_t* stats, float* f_out,
                              float* p_out, int32_t* counts_out, void* stream);

/* ---------------------------------------------------------------------------
 * moe_bias_update -- b[e] += rate * sign(mean(c) - c[e]), optional clamp.
 *
 * Defines: the Practice page's BiasBalancedRouter.update_bias (overloaded experts
 * down, underloaded up, step 1e-3, clamp +-1e-2) and llm-compass "负载均衡".
 * The sign is taken exactly in integers (sum(c) - N c[e]); sign(0) = 0.
 *   counts [N] int32; bias [N] fp32 in/out; clamp <= 0 disables clamping.
 * ------------------------------------------------------------------------- */
int moe_bias_update(const moe_config_t* cfg, const int32_t* counts, float* bias,
                    float rate, float clamp, void* stream);

/* ---------------------------------------------------------------------------
 * moe_bias_update_ema -- the bias controller on a moving average of the loads.
 *
 * The landscape page names an aux-loss-free "bias EMA" controller (TL;DR, §2,
 * 实践要点) without a formula.  Reading: ema <- beta * ema + (1 - beta) * c, then
 * b[e] += rate * sign(mean(ema) - ema[e]) (mean and sign in double), optional
 * clamp.  beta = 0 is moe_bias_update.
 *   counts [N] int32; ema [N] fp32 in/out (caller-owned state, start at 0 or at
 *   the first counts); bias [N] fp32 in/out; 0 <= beta < 1.
 * ------------------------------------------------------------------------- */
int moe_bias_update_ema(const moe_config_t* cfg, const int32_t* counts, float* ema, float beta,
                        float* bias, float rate, float clamp, void* stream);

/* ---------------------------------------------------------------------------
 * moe_bias_update_seq -- bias update on the per-sequence (length-normalised) load.
 *
 * The Practice page's update_bias averages per-sequence statistics so that long
 * sequences do not dominate (its printed mean of raw counts has the same signs as
 * the batch counts); its long-context section suggests weighting by token count.
 * Reading: load[e] = sum over sequences b of c_be / len_b, then
 * b[e] += rate * sign(mean(load) - load[e]) (double), optional clamp.
 *   topk_idx [T, k]; seq_offsets [n_seq+1] int32 (device), token ranges of the
 *   sequences, non-decreasing, seq_offsets[n_seq] <= T; bias [N] in/out;
 *   ws >= 8 * n_seq * N bytes (clobbered).
 * ------------------------------------------------------------------------- */
int moe_bias_update_seq(const moe_config_t* cfg, const int32_t* topk_idx, const int32_t* seq_offsets,
                        int32_t n_seq, float* bias, float rate, float clamp, void* ws,
                        size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Expert-choice routing: moe_route_scores -> moe_expert_choice -> moe_grouped_ffn
 * (G = N, offsets from moe_expert_choice) -> moe_combine_ec.
 *
 * Defines: the Practice page ("路由的数学形式", last paragraphs: each expert picks its
 * top-C tokens by its own capacity; perfectly balanced, no capacity drops; not
 * causal) and the landscape page §0.  Readings: the affinity is the token-choice
 * router's (softmax or sigmoid of x W_g, no bias, no group limit); equal scores go
 * to the lower token index; a picked pair's gate weight is its affinity (no
 * renormalisation); an expert's rows are its picked tokens in ascending order;
 * the caller chooses C (the plain reading is ceil(cf * k * T / N), k being the
 * average number of experts per token).
 * ------------------------------------------------------------------------- */

/* Affinity matrix of the router, expert-major.  scores [N, T] fp32 out;
 * lse [T] and p_partial [nblk, N] as in moe_route; ws as in moe_route.
 * cfg->shared_sink must be 0. */
int moe_route_scores(const moe_config_t* cfg, const void* x, const float* w_gate,
                     const float* logit_offset, float* scores, float* lse, float* p_partial,
                     void* ws, size_t ws_bytes, void* stream);

/* Expert-choice capacity (host out): C = min(T, ceil(cf * k * T / N)) with
 * cf = cfg->capacity_factor (> 0) and k = cfg->top_k read as the average number of
 * experts per token (the Practice page's C = capacity_factor * k * T / n_experts in
 * "容量因子、token dropping"), evaluated as ceil((cf * k * T) / N) in double. */
int moe_expert_choice_capacity(const moe_config_t* cfg, int32_t* capacity);

/* Every expert takes its `capacity` (C, 0 <= C <= T) best tokens.
 *   scores [N, T] (from moe_route_scores); row_of [N, T] int32 out: row of (e, t)
 *   in x_perm or -1; token_of_row [N*C] out; offsets [N+1] out (= e*C);
 *   x_perm [N*C, d] out (x_dtype); n_unpicked [1] int32 or NULL: zeroed here and
 *   counted by moe_combine_ec (tokens no expert picked). */
int moe_expert_choice(const moe_config_t* cfg, const void* x, const float* scores, int32_t capacity,
                      int32_t* row_of, int32_t* token_of_row, int32_t* offsets, void* x_perm,
                      int32_t* n_unpicked, void* stream);

/* y[t] = shared[t] + sum over experts e that picked t (ascending e) of
 * scores[e, t] * y_perm[row_of[e, t]]; fp32 accumulation, no atomics on floats.
 * shared_out [T, d] or NULL; n_unpicked as in moe_expert_choice (or NULL). */
int moe_combine_ec(const moe_config_t* cfg, const void* y_perm, const int32_t* row_of,
                   const float* scores, const void* shared_out, void* y, int32_t* n_unpicked,
                   void* stream);

/* ---------------------------------------------------------------------------
 * moe_permute_noalloc -- moe_permute for callers that cannot allocate.
 *
 * The source pages have no counterpart to this call; it exists for deployment.
 * Some callers cannot allocate device memory: a plugin inside a host
 * application whose memory pool already owns the device, or a runtime with a
 * static memory plan.  This variant computes exactly what moe_permute computes
 * (same outputs, bit for bit) but keeps its per-block count table in a 1 MiB
 * device array inside the library instead of a caller-provided workspace, and
 * calls no allocator.
 *   Arguments: as moe_permute, without ws / ws_bytes (x_perm = NULL skips the
 *   gather, as there).
 *   Limit: ceil(T / 256) * N <= 262144 (e.g. N = 256 up to T = 262144 tokens);
 *          larger calls return MOE_ERR_WORKSPACE_TOO_SMALL and enqueue nothing.
 *   The first call on a device looks up the array's device address (with that
 *   device current), and so does the first call after the device's context has
 *   been replaced (cudaDeviceReset); make those calls before any stream capture.
 *   Every GPU that loads the library holds the array until the process exits.
 *   All calls share the array: calls that overlap on the GPU race, so the
 *   caller must order them (one stream, or explicit events).  Each call
 *   rewrites the table before reading it.
 * ------------------------------------------------------------------------- */
int moe_permute_noalloc(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                        int32_t* counts, int32_t* offsets, int32_t* row_of_slot,
                        int32_t* token_of_row, void* x_perm, int32_t* n_dropped, void* stream);

/* ---------------------------------------------------------------------------
 * Diagnostics.
 * ------------------------------------------------------------------------- */

/* Reads (and, if reset != 0, clears) the device status word of the current
 * device into *status (host out): MOE_OK, MOE_ERR_DEVICE_TIMEOUT (a bounded wait
 * gave up) or MOE_ERR_INVALID_ARG (a kernel met a caller-supplied index outside its
 * range -- an expert id outside [0, N) or repeated within a token, a sequence range
 * outside [0, T] -- and skipped that slot: it is treated as dropped and never
 * dereferenced).  Synchronises the current device. */
int moe_device_status(int32_t* status, int32_t reset);

/* Self-test of the device-side failure detection: launches one thread that waits,
 * through the library's bounded wait, on an mbarrier that can never complete.  The
 * wait gives up after limit_cycles SM clock cycles (1 .. about 2e9), records
 * MOE_ERR_DEVICE_TIMEOUT in the device status word (read it with
 * moe_device_status) and the kernel returns normally, so the context stays usable.
 * completed [1] int32 device out or NULL: 0 when the wait gave up.  No page defines
 * this call: it tests the bounded waits every tensor-core kernel uses. */
int moe_selftest_wait_timeout(int64_t limit_cycles, int32_t* completed, void* stream);

/* Static string for a status code. */
const char* moe_status_string(int status);

/* The CUDA runtime error (cudaError_t value, and its name) behind the last
 * MOE_ERR_CUDA returned to the calling host thread; cudaSuccess / "cudaSuccess" if
 * none.  Host only. */
int moe_last_cuda_error(void);
const char* moe_last_cuda_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */

/*
 * routed_moe.h -- C ABI of libroutedmoe.so: forward pass of a DeepSeek-V3-style
 * routed Mixture-of-Experts block (the LingBot-Video MoE DiT block) on one
 * NVIDIA B200 (sm_100a).
 *
 * What the block computes (sources are web pages, cited by title + section):
 *   [S1] prhub report "sglang PR #32341: LingBot-Video MoE 30B", section
 *        "实现拆解" (implementation breakdown) step 1 and section "关键源码片段"
 *        (key source snippets), LingBotVideoSparseMoeBlock / LingBotVideoRouter.
 *   [S2] xxqk.cn article "vLLM-Omni 原生推理 LingBot-Video", section
 *        "MoE 实现的源码级要点" (source-level MoE notes).
 *
 *   router  : logits = x . Wr^T (fp32), s = sigmoid(logits), c = s + bias;
 *             group score = sum of the top-2 c of each of n_group groups;
 *             keep the topk_group best groups; ids = top_k largest c among
 *             their experts; w = routed_scaling_factor * s[ids] / sum s[ids]
 *             (raw scores, renormalised, scaled once)            [S1] step 1, [S2]
 *   experts : y_e(x) = (silu(x . W13[e,0:I]^T) * (x . W13[e,I:2I]^T)) . W2[e]^T
 *             with w13 packed [E, 2I, H] gate rows then up rows   [S1] snippets
 *   output  : out = sum_i w_i * y_{ids_i}(x) + shared(x) [+ residual]
 *             (fp32 weighted restore; shared expert added unscaled) [S1], [S2]
 *
 * Conventions for every entry point
 *   - Linear layers are y = x . W^T with W row-major [out, in].
 *   - Pointers named "device" are CUDA device memory owned by the caller;
 *     the library never allocates, frees or keeps them.  Host pointers are
 *     only read during the call.
 *   - "stream" is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it and never synchronise the host, except
 *     moe_read_device_status.
 *   - bf16 tensors are IEEE bfloat16, row-major and contiguous.
 *   - Every call checks its arguments first and launches nothing when it
 *     returns an error.  T == 0 is valid and does nothing.
 *   - Calls that share a workspace must not overlap on the device.
 */
#ifndef ROUTED_MOE_H
#define ROUTED_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* null pointer, negative size, inconsistent cfg */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* shape outside what the kernels implement */
  MOE_ERR_WORKSPACE = 3,          /* workspace missing, misaligned or too small */
  MOE_ERR_CUDA = 4,               /* a CUDA runtime / driver call failed */
  MOE_ERR_DEVICE_TIMEOUT = 5,     /* a device-side wait ran past its limit */
  MOE_ERR_DEVICE_INDEX = 6,       /* a kernel met an expert id outside [0, E) */
  MOE_ERR_NO_DEVICE = 7           /* no sm_100 device current */
} moe_status_t;

/* Block configuration.  Defaults of the LingBot-Video MoE model ([S1]
 * "实现拆解" step 3): E=128, I=768, top_k=8, n_group=4, topk_group=2,
 * routed_scaling_factor=2.5, norm_topk_prob=1, one shared expert of I_shared=768. */
typedef struct {
  int32_t T;                      /* tokens (rows of x) */
  int32_t H;                      /* hidden size; multiple of 64 */
  int32_t E;                      /* routed experts; 1..128, divisible by n_group */
  int32_t I;                      /* moe_intermediate_size; multiple of 64 */
  int32_t I_shared;               /* shared expert intermediate size; 0 = none, else multiple of 64 */
  int32_t top_k;                  /* experts per token; 1..16 */
  int32_t n_group;                /* expert groups; 1..16 */
  int32_t topk_group;             /* groups kept per token */
  float routed_scaling_factor;    /* applied once, inside the router */
  int32_t norm_topk_prob;         /* 1: renormalise the chosen scores to sum 1 first */
  int32_t flags;                  /* reserved, must be 0 */
} moe_cfg_t;

/* Stages of moe_forward, in launch order (for stage_events). */
#define MOE_STAGE_ROUTER 0
#define MOE_STAGE_PERMUTE 1
#define MOE_STAGE_EXPERT_UP 2
#define MOE_STAGE_EXPERT_DOWN 3
#define MOE_STAGE_SHARED_EXPERT 4
#define MOE_STAGE_COMBINE 5
#define MOE_NUM_STAGES 6

/* Optional arguments of moe_forward (pass NULL for all defaults). */
typedef struct {
  const void* residual;   /* device bf16 [T,H] or NULL: out = residual + block(x);
                             may be the same buffer as out */
  int32_t* topk_ids;      /* device int32 [T,top_k] or NULL: also write the routing ids */
  float* topk_w;          /* device fp32 [T,top_k] or NULL: also write the routing weights */
  void** stage_events;    /* host array of MOE_NUM_STAGES+1 cudaEvent_t or NULL: event i (if
                             not NULL) is recorded on stream before stage i, the last one after
                             the last stage.  Each recorded event orders the kernels around it
                             strictly, so record only the boundaries you time. */
  int64_t wait_timeout_ns;/* limit of every device-side wait; 0 = 2 s */
  const uint8_t* token_mask; /* device uint8 [T] or NULL (all real): padding mask ([S2] "MoE
                             实现的源码级要点": the mask acts on the routing scores, which are
                             renormalised); a token with mask 0 takes no routed expert (id -1,
                             weight 0) and its output is the shared expert (+ residual) */
} moe_forward_opts_t;

/* Human-readable name of a status code; never NULL. */
MOE_API const char* moe_status_string(int32_t status);

/* Checks cfg against the limits above; MOE_OK or the first violation.
 * [S1] "风险与影响" item 4 names the divisibility of E by n_group and a
 * group of at least 2 experts (the per-group top-2) as assumptions. */
MOE_API int32_t moe_check_config(const moe_cfg_t* cfg);

/* Workspace bytes needed by moe_route / moe_permute / moe_forward for cfg
 * (0 when cfg is invalid).  The workspace is device memory, 256-byte aligned. */
MOE_API size_t moe_route_workspace_bytes(const moe_cfg_t* cfg);
MOE_API size_t moe_permute_workspace_bytes(const moe_cfg_t* cfg);
MOE_API size_t moe_workspace_bytes(const moe_cfg_t* cfg);

/* Router ([S1] step 1, LingBotVideoRouter.forward(tokens) -> (top_indices,
 * top_scores); [S2] asymmetric routing).
 *   x        device bf16 [T,H]
 *   Wr       device fp32 [E,H]   router weight (kept in fp32)
 *   bias     device fp32 [E]     e_score_correction_bias (selection only)
 *   topk_ids device int32 [T,top_k] out: expert ids, descending c, ties to the lower id
 *   topk_w   device fp32 [T,top_k] out: gating weights, same order
 *   workspace device, moe_route_workspace_bytes(cfg) bytes, 256-byte aligned:
 *            status word, the bf16 three-term split of Wr and fp32 partial logits. */
MOE_API int32_t moe_route(const void* x, const float* Wr, const float* bias, const moe_cfg_t* cfg,
                  int32_t* topk_ids, float* topk_w, void* workspace, size_t workspace_bytes,
                  void* stream);

/* moe_route with a per-token padding mask ([S2] "MoE 实现的源码级要点": the
 * padding mask acts on the routing scores, which are renormalised):
 *   token_mask device uint8 [T]: 0 = padding.  A padding token's routing
 *              scores are masked to zero, so it takes no expert: its ids are
 *              -1 and its weights 0 (an all-zero row stays zero when
 *              renormalised).  Real tokens are routed exactly as by moe_route.
 * Other arguments, workspace and errors as moe_route; token_mask NULL is
 * moe_route. */
MOE_API int32_t moe_route_masked(const void* x, const float* Wr, const float* bias,
                                 const uint8_t* token_mask, const moe_cfg_t* cfg,
                                 int32_t* topk_ids, float* topk_w, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Token -> expert permutation ([S2] "_reorder_tokens": tokens regrouped per
 * expert before the grouped GEMMs).  Rows are ordered by expert, then by
 * token, so the permutation is unique and deterministic.
 *   topk_ids       device int32 [T,top_k], every id in [0,E)
 *   topk_w         device fp32 [T,top_k] or NULL
 *   x              device bf16 [T,H] or NULL (then xp is not written)
 *   expert_offsets device int32 [E+1] out: first row of each expert, [E] = T*top_k
 *   row_of         device int32 [T*top_k] out: row of (token t, slot j) at t*top_k+j
 *   tok_of         device int32 [T*top_k] out: token of each row
 *   w_of           device fp32 [T*top_k] out or NULL: weight of each row
 *   xp             device bf16 [T*top_k, H] out or NULL: xp[row] = x[tok_of[row]]
 * An id outside [0,E) is skipped and leaves MOE_ERR_DEVICE_INDEX in the
 * workspace status word (see moe_read_device_status). */
MOE_API int32_t moe_permute(const int32_t* topk_ids, const float* topk_w, const void* x,
                    const moe_cfg_t* cfg, int32_t* expert_offsets, int32_t* row_of,
                    int32_t* tok_of, float* w_of, void* xp, void* workspace,
                    size_t workspace_bytes, void* stream);

/* Largest T that moe_permute_noalloc accepts. */
#define MOE_NOALLOC_MAX_T 65536

/* moe_permute without a workspace argument: the same permutation, bit for
 * bit, for callers that cannot allocate device memory themselves -- for
 * example an operator running inside another framework that hands it its
 * inputs and outputs and owns every device allocation, or a latency-critical
 * loop where a cudaMalloc (which can synchronise the device) is not allowed.
 * The source pages have no counterpart to this entry point.
 *   Arguments are those of moe_permute minus workspace / workspace_bytes.
 *   Scratch: a fixed array of about 129 KiB in the library's device memory,
 *   one copy on every GPU that loads the library, held until the process
 *   exits.  T > MOE_NOALLOC_MAX_T returns MOE_ERR_UNSUPPORTED_SHAPE and
 *   launches nothing.  The call allocates nothing (no cudaMalloc/cudaFree).
 *   The first call on a device looks up the array's device address (once
 *   per device, with that device current); make that first call before any
 *   stream capture.  A device reset (cudaDeviceReset) frees the array with
 *   the device's context; the next call sees a new context and looks the
 *   address up again, so it also belongs before any capture.
 *   Every call on a device shares the one array and it keeps the last call's
 *   contents: calls that overlap on the GPU (different streams, no ordering)
 *   race and give wrong results.  An expert id outside [0,E) is skipped and
 *   its row_of entry set to -1 (the status word is not exposed). */
MOE_API int32_t moe_permute_noalloc(const int32_t* topk_ids, const float* topk_w, const void* x,
                                    const moe_cfg_t* cfg, int32_t* expert_offsets,
                                    int32_t* row_of, int32_t* tok_of, float* w_of, void* xp,
                                    void* stream);

/* Whole block forward ([S1] LingBotVideoSparseMoeBlock.forward: router ->
 * grouped SwiGLU experts with the router weight applied on the output ->
 * fp32 restore ([S2] "_restore_tokens") -> + shared expert, unscaled).
 *   x     device bf16 [T,H]          block input
 *   Wr    device fp32 [E,H], bias device fp32 [E]
 *   w13   device bf16 [E,2I,H]       gate rows 0..I-1, up rows I..2I-1 (non-interleaved)
 *   w2    device bf16 [E,H,I]
 *   ws13  device bf16 [2I_s,H], ws2 device bf16 [H,I_s]  (NULL when I_shared == 0)
 *   out   device bf16 [T,H]          must not overlap x
 *   opts  host pointer or NULL
 * Each expert output (router weight applied in fp32) is stored as bf16; the
 * restore sums them in fp32 in a fixed order (slots 0..top_k-1, then the
 * shared expert, then the residual) and rounds once, so the result is
 * bitwise reproducible and each token's output does not depend on the other
 * tokens of the call. */
MOE_API int32_t moe_forward(const void* x, const float* Wr, const float* bias, const void* w13,
                    const void* w2, const void* ws13, const void* ws2, const moe_cfg_t* cfg,
                    void* out, const moe_forward_opts_t* opts, void* workspace,
                    size_t workspace_bytes, void* stream);

/* moe_forward with FP8 expert weights.  The pages name an optional FP8
 * backend of the upstream project ([S3] "Known limitations") without a
 * format; this entry point takes weight-only FP8: every expert matrix as OCP
 * E4M3 codes ("fn": no infinities) with one power-of-two scale per 128 x 128
 * block, given as a UE8M0 byte s (scale 2^(s-127)).  Weights are dequantised
 * to bf16 in shared memory next to the tensor cores; with power-of-two
 * scales the dequantised weights are exact bf16 values, so the result is bit
 * for bit that of moe_forward on the dequantised bf16 weights.
 *   w13_q  device uint8 [E,2I,H]  E4M3 codes, gate rows then up rows
 *   w13_s  device uint8 [E,2I/128,H/128]  scale exponents
 *   w2_q   device uint8 [E,H,I];  w2_s device uint8 [E,H/128,I/128]
 *   ws13_q / ws13_s  [2I_s,H] / [2I_s/128,H/128];  ws2_q / ws2_s  [H,I_s] /
 *          [H/128,I_s/128]  the shared expert (NULL when I_shared == 0)
 * H, I and I_shared must be multiples of 128 (MOE_ERR_UNSUPPORTED_SHAPE);
 * scale exponents 255 (NaN) and E4M3 NaN codes are not checked and give
 * undefined values.  Workspace: moe_workspace_bytes(cfg).  Every other
 * argument, option and error as moe_forward.  The expert GEMMs run with
 * swapped operands (weight rows on the MMA's M) at every batch size. */
MOE_API int32_t moe_forward_fp8(const void* x, const float* Wr, const float* bias,
                                const uint8_t* w13_q, const uint8_t* w13_s,
                                const uint8_t* w2_q, const uint8_t* w2_s,
                                const uint8_t* ws13_q, const uint8_t* ws13_s,
                                const uint8_t* ws2_q, const uint8_t* ws2_s,
                                const moe_cfg_t* cfg, void* out, const moe_forward_opts_t* opts,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of moe_forward_host: those of moe_forward plus four
 * [T,H] bf16 staging buffers (two for inputs, two for outputs); 0 for an
 * invalid configuration. */
MOE_API size_t moe_forward_host_workspace_bytes(const moe_cfg_t* cfg);

/* moe_forward over n_batches independent batches of cfg->T tokens that live
 * in HOST memory: batch b is copied in from x_host[b], run through the block
 * (the same kernels and bits as moe_forward, no residual) and copied out to
 * out_host[b].  The sources define only the block itself; streaming
 * host-resident batches through it, with the copies of the neighbouring
 * batches overlapping each batch's kernels, is this library's own addition.
 *   x_host, out_host  host arrays of n_batches host pointers, each to a
 *                     [T,H] bf16 row-major batch; a pointer may repeat (the
 *                     same input several times, one output buffer reused),
 *                     but no output may overlap any input.
 *                     Page-locked memory (cudaHostAlloc / cudaHostRegister)
 *                     lets the copies overlap the kernels; pageable memory
 *                     gives the same results with the copies serialised.
 *   Wr ... ws2        device weights, as for moe_forward
 *   workspace         device, moe_forward_host_workspace_bytes(cfg) bytes,
 *                     256-byte aligned
 *   stream            runs the kernels; h2d_stream / d2h_stream run the
 *                     copies in / out (NULL: stream itself, no overlap).
 * Everything starts after the work already queued on stream, and work queued
 * on stream after this call starts only once every out_host[b] is written;
 * the host buffers must stay valid until then.  Batches run in order; inputs
 * are double-buffered so that batch b+1 is copied in while batch b computes
 * and batch b-1 is copied out.  The status word is cleared by the first
 * batch only, so moe_read_device_status reports the first device-side error
 * of any batch.  Host checks (as moe_forward, plus n_batches < 0, a NULL
 * batch pointer or an output overlapping an input) launch nothing; a CUDA
 * failure part-way returns MOE_ERR_CUDA with the earlier batches queued. */
MOE_API int32_t moe_forward_host(const void* const* x_host, void* const* out_host,
                                 int32_t n_batches, const float* Wr, const float* bias,
                                 const void* w13, const void* w2, const void* ws13,
                                 const void* ws2, const moe_cfg_t* cfg, void* workspace,
                                 size_t workspace_bytes, void* stream, void* h2d_stream,
                                 void* d2h_stream);

/* Dense feed-forward layer ([S2] "MoE 实现的源码级要点": a transformer block
 * uses the sparse MoE block or a plain LingBotVideoMLP -- the dense FFN -- by
 * decoder_sparse_step and layer index; the shared expert is the same MLP):
 *   out = bf16( [residual +] SwiGLU(x) ),  SwiGLU(x) = (silu(x.Wg^T) * (x.Wu^T)) . W2^T
 *   x        device bf16 [T,H]
 *   w13      device bf16 [2I,H]   gate rows 0..I-1, up rows I..2I-1 (non-interleaved)
 *   w2       device bf16 [H,I]
 *   residual device bf16 [T,H] or NULL; may be the same buffer as out
 *   out      device bf16 [T,H], must not overlap x
 *   workspace device, moe_dense_ffn_workspace_bytes(T,H,I) bytes, 256-byte aligned
 * H and I multiples of 64 (<= 16384).  The intermediate h is stored in bf16;
 * with a residual the MLP output is stored in bf16 and added to the residual
 * in fp32 with one final rounding (as the block's restore).  Device-side
 * errors go to the workspace status word (moe_read_device_status). */
MOE_API size_t moe_dense_ffn_workspace_bytes(int32_t T, int32_t H, int32_t I);
MOE_API int32_t moe_dense_ffn(const void* x, const void* w13, const void* w2, int32_t T,
                              int32_t H, int32_t I, const void* residual, void* out,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- expert parallelism
 * Building blocks of the block with its experts split across ranks (one GPU
 * per rank): every rank routes and permutes its own tokens (moe_route,
 * moe_permute: the rows for each rank's experts are then contiguous), sends
 * the rows, their expert ids (moe_rows_expert_ids) and router weights to the
 * ranks that hold those experts, which sort them by expert (moe_permute with
 * top_k = 1) and run moe_expert_rows; the results come back to the tokens'
 * ranks, which restore each token with moe_combine_rows and the shared expert
 * (moe_dense_ffn on their own tokens).  The exchange itself is the caller's
 * (an all-to-all each way).  The arithmetic of every row and of the restore is
 * the block's own ([S1] LingBotVideoSparseMoeBlock.forward; [S2] the fp32
 * restore), so the result is bit for bit that of moe_forward; the pages state
 * no expert-parallel form ([S3] "Known limitations": no expert parallelism is
 * claimed), and this split is the library's own. */

/* ids[r] (device int32 [R]) = the expert e whose rows [offsets[e], offsets[e+1])
 * contain row offsets[0] + r; offsets device int32 [E+1], non-decreasing,
 * R = offsets[E] - offsets[0].  E in 1..128. */
MOE_API int32_t moe_rows_expert_ids(const int32_t* offsets, int32_t E, int32_t R, int32_t* ids,
                                    void* stream);

/* Workspace bytes of moe_expert_rows; 0 for invalid sizes. */
MOE_API size_t moe_expert_rows_workspace_bytes(int32_t R, int32_t H, int32_t E, int32_t I);

/* The routed experts on rows already grouped by expert: for expert e (0..E-1)
 * and each row r in [offsets[e], offsets[e+1]):
 *   y[row_dest[r]] = bf16( row_w[r] * (silu(x_r.Wg_e^T) * (x_r.Wu_e^T)) . W2_e^T )
 * with h stored in bf16 and the weight applied in fp32, as in moe_forward.
 *   xr       device bf16 [R,H]; offsets device int32 [E+1], offsets[0] >= 0,
 *            offsets[E] <= R (rows outside the groups are not computed)
 *   w13      device bf16 [E,2I,H] (gate rows, then up rows); w2 device bf16 [E,H,I]
 *   row_w    device fp32 [R] (NULL: 1); row_dest device int32 [R], distinct rows of y
 *   y        device bf16 [>= max(row_dest)+1, H]
 * E in 1..128; H and I multiples of 64 (<= 16384).  Workspace:
 * moe_expert_rows_workspace_bytes(R,H,E,I), 256-byte aligned; device-side errors
 * go to its status word (moe_read_device_status). */
MOE_API int32_t moe_expert_rows(const void* xr, const int32_t* offsets, int32_t R, int32_t E,
                                int32_t H, int32_t I, const void* w13, const void* w2,
                                const float* row_w, const int32_t* row_dest, void* y,
                                void* workspace, size_t workspace_bytes, void* stream);

/* The restore with each token's routed rows addressed through row_of:
 *   out[t] = bf16( sum_{j<top_k} y[row_of[t*top_k+j]] [+ shared[t]] [+ residual[t]] )
 * summed in fp32 in that order, rounded once -- the order and rounding of
 * moe_forward's restore ([S2] "_restore_tokens").  A row_of entry outside
 * [0, R) adds 0, like a rejected expert id (there is no status word here: such
 * an entry is not reported).
 *   y device bf16 [R,H]; row_of device int32 [T,top_k]; shared, residual
 *   device bf16 [T,H] or NULL; out device bf16 [T,H] (may be residual).
 * H a multiple of 64 (<= 16384); top_k in 1..16; R >= 0. */
MOE_API int32_t moe_combine_rows(const void* y, int32_t R, const int32_t* row_of, int32_t T,
                                 int32_t H, int32_t top_k, const void* shared,
                                 const void* residual, void* out, void* stream);

/* RMSNorm with fp32 accumulation ([S2]: RMSNorm accumulates in fp32), for a
 * residual stack of blocks: xn = bf16(x * rsqrt(mean(x^2) + eps) * gamma).
 *   x device bf16 [T,H]; gamma device fp32 [H] or NULL (= 1); xn device bf16 [T,H]. */
MOE_API int32_t moe_rmsnorm(const void* x, const float* gamma, float eps, int32_t T, int32_t H,
                    void* xn, void* stream);

/* Waits for stream, then reads and clears the device status word that the
 * kernels of moe_forward / moe_permute leave in workspace (MOE_OK, or the
 * first device-side error of the last call).  *site receives where the
 * error arose (kernel-specific; may be NULL). */
MOE_API int32_t moe_read_device_status(void* workspace, int32_t* site, void* stream);

/* Failure-detection self test: launches one kernel whose thread waits on a
 * device flag that nothing sets, with the same bounded wait that every
 * pipeline wait of the library uses.  The wait gives up after timeout_ns and
 * leaves MOE_ERR_DEVICE_TIMEOUT in the status word of workspace (>= 256 bytes);
 * the context stays usable. */
MOE_API int32_t moe_selftest_wait_timeout(void* workspace, int64_t timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ROUTED_MOE_H */

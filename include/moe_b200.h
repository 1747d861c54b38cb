/*
 * moe_b200.h -- C ABI of the sparse Mixture-of-Experts FFN layer forward on
 * one NVIDIA B200 (sm_100a).
 *
 * What the layer computes (reference pages, cited by title and section):
 *   "論文解説: DeepSeekMoE — 細粒度エキスパート分割と共有エキスパートによるMoE効率化"
 *     §ルーティングとバランス損失: s_j = softmax(W_r x)_j over all routed
 *       experts, g_j = s_j / sum_{k in TopK} s_k, balance term
 *       alpha * N_r * sum_j f_j P_j;
 *     §共有エキスパート機構: h_t = sum_i E_s,i(x_t) + sum_{j in TopK} g_j E_r,j(x_t);
 *     §アルゴリズム: router = Linear without bias; each expert
 *       Linear(d, d_ff) + bias -> SiLU -> Linear(d_ff, d) + bias.
 *   "Sparse MoE Top-Kルーティング" §ルーティングの仕組み (top-K, gate weights),
 *     §解決策2 and FAQ Q2 (per-expert capacity per batch; overflow dropped).
 *   "エキスパート並列（Expert Parallelism）" §推論フロー: tokens travel to their
 *     expert and back; on one GPU this exchange is an on-device permutation
 *     (moe_dispatch / moe_combine).
 *   "DeepSeek DeepEP" §DeepEP とは item 5, §DeepEP の性能: FP8 dispatch,
 *     BF16 combine.
 *
 * Readings fixed by this library where the pages are silent:
 *   - top-K is taken on the fp32 logits; equal logits go to the lower expert
 *     index; slot k = 0..K-1 is in descending logit order;
 *   - capacity C = ceil(capacity_factor * T * K / N_r), evaluated exactly on
 *     the fp32 capacity_factor; within an expert the slots keep token order
 *     and the first C are kept; a dropped slot contributes nothing and the
 *     other gates are not renormalised;
 *   - f_j = counts_j / (T*K) with pre-drop counts; P_j = mean over all T
 *     tokens of the full softmax (after any logit bias);
 *   - FP8: e4m3 codes, activations with one fp32 scale per row per 128
 *     columns, weights with one fp32 scale per 128x128 block; every scale the
 *     library produces is the smallest power of two 2^k with
 *     amax / 2^k <= 448 (1 for an all-zero block), codes round to nearest
 *     even and saturate to +-448.  The hidden activation is re-quantised the
 *     same way between the two linear layers; expert outputs are bf16.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE memory owned by the caller, row-major
 *     and densely packed.  The library allocates nothing, keeps no state
 *     between calls and never synchronises the host (except
 *     moe_get_device_status).  `stream` is a cudaStream_t (NULL = legacy
 *     default stream); every call is asynchronous on it.
 *   - Tokens are flattened: x is (T, d_model).  Activation dtype: fp32
 *     (MOE_F32) or bf16 (MOE_BF16, MOE_FP8_E4M3_BLOCK).  Router weight W_r is
 *     fp32 (N_r, d_model) in every mode.  Biases are fp32.
 *   - Expert weights are stacked and K-contiguous: W1 (N_r, d_ff, d_model),
 *     W2 (N_r, d_model, d_ff), shared Ws1 (n_shared, d_ff_shared, d_model),
 *     Ws2 (n_shared, d_model, d_ff_shared); dtype fp32, bf16, or e4m3 bytes in
 *     FP8 mode with fp32 block scales W*_scales (E, rows/128, cols/128).
 *   - `ws` is a caller-allocated workspace of moe_workspace_size() bytes,
 *     256-byte aligned.  It must be zero-filled once before first use
 *     (moe_workspace_init); afterwards calls keep it consistent.  Stages
 *     communicate through it (moe_route -> moe_balance_stats), so one ws
 *     must not be shared by calls that overlap on the GPU.
 *   - Row counts: R_cap = T*K without a capacity, else min(T*K, N_r*C).
 *     moe_buffer_rows() returns C, R_cap and the row counts of x_disp and y.
 *   - Every call returns MOE_OK or an error code.  Argument errors are found
 *     on the host before anything is launched.  Errors found by kernels
 *     (bad routing indices, a bounded wait that expired) are OR-ed into a
 *     status word inside ws and read with moe_get_device_status().
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_EXPORT __attribute__((visibility("default")))
#else
#define MOE_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes -------------------------------------------------------- */
#define MOE_OK                 0
#define MOE_ERR_INVALID_ARG    1  /* null pointer, bad size, misaligned pointer */
#define MOE_ERR_UNSUPPORTED    2  /* shape outside what the kernels handle      */
#define MOE_ERR_CUDA           3  /* a CUDA call failed; see moe_last_cuda_error */
#define MOE_ERR_BAD_ROUTING    4  /* device: topk_idx out of range or repeated   */
#define MOE_ERR_DEVICE_TIMEOUT 5  /* device: a bounded wait expired              */

/* device status word bits (moe_get_device_status) */
#define MOE_DEV_BAD_ROUTING    0x1
#define MOE_DEV_TIMEOUT        0x2

/* ---- dtypes ---------------------------------------------------------------- */
#define MOE_F32             0   /* fp32 activations and weights                  */
#define MOE_BF16            1   /* bf16 activations and weights, fp32 accumulate */
#define MOE_FP8_E4M3_BLOCK  2   /* e4m3 dispatch + weights with block scales,
                                   bf16 expert outputs and layer output          */

/* Layer shape.  Mirrors the reference module's constructor
 * (d_model, n_routed, n_shared, top_k, d_ff) plus the batch size, the shared
 * experts' width, the capacity factor and the balance weight alpha. */
typedef struct {
    int32_t T;               /* tokens in the batch (B*S), >= 1                   */
    int32_t d_model;         /* hidden size d                                     */
    int32_t n_routed;        /* N_r routed experts, 1..256                        */
    int32_t top_k;           /* K experts per token, 1..min(N_r, 16)              */
    int32_t d_ff;            /* routed expert FFN width                           */
    int32_t n_shared;        /* K_s always-on shared experts, 0..8                */
    int32_t d_ff_shared;     /* shared expert FFN width (ignored if n_shared==0)  */
    float   capacity_factor; /* 0 = no capacity limit                             */
    float   alpha;           /* balance weight (the pages recommend 0.01)         */
    int32_t dtype;           /* MOE_F32 | MOE_BF16 | MOE_FP8_E4M3_BLOCK           */
    int32_t bias_mode;       /* how logit_bias is used (see MOE_BIAS_*)           */
    int32_t capacity_priority; /* which slots an expert keeps (MOE_PRIORITY_*)   */
    int32_t overflow_mode;   /* what a slot over the capacity gives (MOE_OVERFLOW_*) */
} moe_config;

/* capacity_priority ("Sparse MoE Top-Kルーティング" §解決策2, FAQ Q2).
 * MOE_PRIORITY_TOKEN: an expert's slots are ranked in token order and the
 * first C are kept (the earliest tokens).  MOE_PRIORITY_SLOT: every token's
 * first choice ranks before any second choice (then token order), so a
 * token's top expert is dropped last.  Rows of an expert's segment follow the
 * rank order. */
#define MOE_PRIORITY_TOKEN  0
#define MOE_PRIORITY_SLOT   1

/* overflow_mode (same section: tokens over the capacity are dropped or passed
 * through).  MOE_OVERFLOW_DROP: a dropped slot adds nothing.
 * MOE_OVERFLOW_PASS: a dropped slot adds gate * x[t], the token's own input
 * (it passes that expert unchanged); moe_combine then needs x. */
#define MOE_OVERFLOW_DROP   0
#define MOE_OVERFLOW_PASS   1

/* bias_mode.  MOE_BIAS_LOGITS: the per-expert bias is added to the router
 * logits, so softmax, top-K, gates and P all see it.  MOE_BIAS_SELECTION:
 * the bias enters only the top-K keys (l + b); softmax, gates and P use the
 * unbiased logits -- the auxiliary-loss-free balancing of "Sparse MoE
 * Top-Kルーティング" §解決策3, where a per-expert bias steers which experts
 * are chosen without changing the loss (the pages give no formula; this is
 * the plainest reading).  logits_out holds the softmax logits (l + b, or l). */
#define MOE_BIAS_LOGITS     0
#define MOE_BIAS_SELECTION  1

/* ---- sizing helpers (host only, no GPU work) ------------------------------ */

/* Validates cfg and returns the workspace size in bytes for any entry point
 * of this header (the largest user is moe_layer_forward).
 * Errors: MOE_ERR_INVALID_ARG (null or inconsistent cfg),
 * MOE_ERR_UNSUPPORTED (d_model or d_ff not a multiple of 64 in bf16 mode or
 * of 128 in FP8 mode, n_routed > 256, top_k > 16, n_shared > 8). */
MOE_EXPORT int moe_workspace_size(const moe_config* cfg, size_t* bytes);

/* capacity: C, or -1 without a limit.  r_cap: R_cap.
 * x_disp_rows: rows of moe_dispatch's x_disp = R_cap, plus T in FP8 mode
 * with shared experts (those T rows carry the quantised x for them).
 * y_rows: rows of moe_expert_ffn's y = R_cap + n_shared*T. */
MOE_EXPORT int moe_buffer_rows(const moe_config* cfg, int32_t* capacity, int32_t* r_cap,
                    int32_t* x_disp_rows, int32_t* y_rows);

/* Zero-fills ws (status word and every counter) on `stream`. */
MOE_EXPORT int moe_workspace_init(const moe_config* cfg, void* ws, void* stream);

/* Synchronises `stream`, then returns in *status the device status word of ws
 * (MOE_DEV_* bits, 0 = clean).  If clear != 0 the word is reset to 0. */
MOE_EXPORT int moe_get_device_status(const moe_config* cfg, void* ws, void* stream,
                          int32_t* status, int32_t clear);

/* The cudaError_t of the last failed CUDA call made by this library on the
 * calling thread (0 if none). */
MOE_EXPORT int moe_last_cuda_error(void);

/* Human-readable name of a MOE_* status code (static string). */
MOE_EXPORT const char* moe_status_string(int status);

/* Number of CUDA kernels this library has launched in this process, on every
 * device and stream, since it was loaded (a launch counts when it is issued,
 * whether or not it later fails).  Thread-safe; read it before and after a
 * sequence of calls to learn how many kernels the sequence launched.  Not a
 * step of the method: bookkeeping for benchmarks. */
MOE_EXPORT uint64_t moe_kernel_launches(void);

/* ---- stage 1: router ------------------------------------------------------
 * l[t,j] = sum_i x[t,i] W_r[j,i] (+ logit_bias[j] with MOE_BIAS_LOGITS) in
 * fp32; s = softmax(l); topk_idx[t,k] = the K largest keys l (+ logit_bias[j]
 * with MOE_BIAS_SELECTION, added in fp32), ties -> lower j, descending;
 * gates[t,k] = s[t,topk_idx[t,k]] / sum_k' s[t,topk_idx[t,k']].
 * Also writes per-block partial sums of s into ws for moe_balance_stats.
 *   x          (T, d_model) fp32 (MOE_F32) or bf16
 *   W_r        (N_r, d_model) fp32
 *   logit_bias (N_r) fp32 or NULL
 *   topk_idx   (T, K) int32 out;  gates (T, K) fp32 out
 *   logits_out (T, N_r) fp32 out, or NULL
 * Pointers must be 16-byte aligned. */
MOE_EXPORT int moe_route(const moe_config* cfg, const void* x, const float* W_r,
              const float* logit_bias, int32_t* topk_idx, float* gates,
              float* logits_out, void* ws, void* stream);

/* ---- stage 2: dispatch ----------------------------------------------------
 * counts[j] = #slots selecting expert j (pre-drop); kept[j] = min(counts, C);
 * offsets (N_r+1) = exclusive prefix sum of kept; slot_row[t,k] = row of
 * slot (t,k) in x_disp (in capacity-rank order within an expert's segment:
 * ascending t, or slot-major with MOE_PRIORITY_SLOT), -1 if dropped by the
 * capacity, -2 if its expert index is invalid; row_slot[r] = t*K+k for
 * r < offsets[N_r].
 * x_disp receives x[t] for every kept slot: as-is in fp32/bf16 mode; in FP8
 * mode as e4m3 codes with x_disp_scales (rows, d_model/128) fp32, plus (with
 * shared experts) the quantised x of every token at rows R_cap..R_cap+T-1.
 * A topk_idx entry outside [0, N_r) or repeated within a token sets
 * MOE_DEV_BAD_ROUTING; such slots are dropped.
 *   x_disp  (x_disp_rows, d_model); x_disp_scales NULL unless FP8. */
MOE_EXPORT int moe_dispatch(const moe_config* cfg, const void* x, const int32_t* topk_idx,
                 int32_t* counts, int32_t* kept, int32_t* offsets,
                 int32_t* slot_row, int32_t* row_slot, void* x_disp,
                 float* x_disp_scales, void* ws, void* stream);

/* ---- stage 3: expert FFNs (grouped GEMMs) ---------------------------------
 * For every routed expert e and its rows r in [offsets[e], offsets[e+1]):
 *   y[r] = W2_e SiLU(W1_e x_disp[r] + b1_e) + b2_e;
 * for every shared expert s and token t:
 *   y[R_cap + s*T + t] = Ws2_s SiLU(Ws1_s x[t] + bs1_s) + bs2_s
 * (in FP8 mode the shared experts read the quantised x from x_disp rows
 * R_cap..R_cap+T-1, and the hidden activation is re-quantised to e4m3 per
 * row per 128 columns before the second layer).  The hidden activations live
 * in ws.  y is (y_rows, d_model): fp32 in MOE_F32 mode, bf16 otherwise.
 * Rows of y beyond offsets[N_r] and below R_cap are not written.
 * Scale pointers are NULL unless FP8; shared-expert pointers are NULL when
 * n_shared == 0. */
MOE_EXPORT int moe_expert_ffn(const moe_config* cfg, const void* x, const void* x_disp,
                   const float* x_disp_scales, const int32_t* offsets,
                   const void* W1, const float* W1_scales, const float* b1,
                   const void* W2, const float* W2_scales, const float* b2,
                   const void* Ws1, const float* Ws1_scales, const float* bs1,
                   const void* Ws2, const float* Ws2_scales, const float* bs2,
                   void* y, void* ws, void* stream);

/* ---- stage 3 over caller-made segments (expert parallelism) ----------------
 * The grouped expert FFN of moe_expert_ffn over n_seg segments of x_rows that
 * the caller lays out: rows seg_offsets[i] .. seg_offsets[i+1]-1 go through
 * expert seg_expert[i] (0 <= seg_expert[i] < n_routed), and y row r is the
 * output of x_rows row r.  Segments may name an expert more than once and in
 * any order: an expert-parallel rank runs its experts on the rows every
 * source rank sent it, in the order they arrived (one segment per source rank
 * and expert), without regrouping them ("エキスパート並列（Expert
 * Parallelism）" §推論フロー: each GPU computes the tokens routed to the
 * experts it holds; "DeepSeek DeepEP" §DeepEP とは: FP8 dispatch, the rows
 * arrive as e4m3 codes with their 1x128 scales).
 *   cfg         n_routed = the experts held, top_k = 1, T = rows of x_rows and
 *               y, n_shared = 0, no capacity (capacity_factor 0); d_model,
 *               d_ff and dtype as the layer's
 *   x_rows      (T, d_model) fp32 / bf16 rows, or e4m3 codes (FP8)
 *   x_rows_scales (T, d_model/128) fp32 (FP8), else NULL
 *   seg_offsets (n_seg+1) int32 device, non-decreasing, seg_offsets[n_seg] <= T
 *   seg_expert  (n_seg) int32 device; 1 <= n_seg <= 256
 *   W1 .. b2    the held experts' weights, as moe_expert_ffn
 *   y           (T, d_model) fp32 (MOE_F32) or bf16; rows outside every
 *               segment are not written
 *   ws          moe_workspace_size(cfg) bytes (hidden activations, status word)
 * A segment whose bounds lie outside [0, T] or whose expert is out of range is
 * skipped and sets MOE_DEV_BAD_ROUTING in ws's status word.  Other argument
 * errors return MOE_ERR_INVALID_ARG before anything is enqueued. */
MOE_EXPORT int moe_expert_ffn_segments(const moe_config* cfg, const void* x_rows,
                   const float* x_rows_scales, const int32_t* seg_offsets,
                   const int32_t* seg_expert, int32_t n_seg,
                   const void* W1, const float* W1_scales, const float* b1,
                   const void* W2, const float* W2_scales, const float* b2,
                   void* y, void* ws, void* stream);

/* ---- stage 4: combine ------------------------------------------------------
 * out[t] = sum_{k ascending, slot_row[t,k] >= 0} gates[t,k] * y[slot_row[t,k]]
 *          (+ gates[t,k] * x[t] for slot_row[t,k] == -1 with MOE_OVERFLOW_PASS)
 *          + sum_{s ascending} y[R_cap + s*T + t], accumulated in fp32.
 * x (T, d_model), as given to moe_dispatch: read only with MOE_OVERFLOW_PASS
 * (may be NULL otherwise).
 * out (T, d_model) fp32 (MOE_F32) or bf16 (round-to-nearest-even). */
MOE_EXPORT int moe_combine(const moe_config* cfg, const void* y, const float* gates,
                const int32_t* slot_row, const void* x, void* out, void* stream);

/* ---- stage 5: balance statistics ------------------------------------------
 * f[j] = counts[j] / (T*K); P[j] = (1/T) sum_t s[t,j] from the partial sums
 * moe_route left in ws; loss = alpha * N_r * sum_j f[j] P[j].  Reductions run
 * in a fixed order (bit-reproducible). f, P (N_r) fp32, loss (1) fp32. */
MOE_EXPORT int moe_balance_stats(const moe_config* cfg, const int32_t* counts,
                      const void* ws, float* f, float* P, float* loss,
                      void* stream);

/* ---- the whole layer --------------------------------------------------------
 * Runs route -> dispatch -> expert FFNs -> combine -> balance statistics on
 * `stream` with every intermediate in ws.  out (T, d_model) as moe_combine;
 * f, P, loss as moe_balance_stats (non-NULL).  topk_idx, gates (T, K) and
 * counts (N_r) receive the routing when non-NULL. */
MOE_EXPORT int moe_layer_forward(const moe_config* cfg, const void* x, const float* W_r,
                      const float* logit_bias,
                      const void* W1, const float* W1_scales, const float* b1,
                      const void* W2, const float* W2_scales, const float* b2,
                      const void* Ws1, const float* Ws1_scales, const float* bs1,
                      const void* Ws2, const float* Ws2_scales, const float* bs2,
                      void* out, float* f, float* P, float* loss,
                      int32_t* topk_idx, float* gates, int32_t* counts,
                      void* ws, void* stream);

/* ---- self-test of the bounded-wait path ------------------------------------
 * Launches one block that waits on an mbarrier which nothing completes, with
 * a wait limit of timeout_ns nanoseconds (clamped to [1e3, 1e10]); the wait
 * gives up, the kernel records MOE_DEV_TIMEOUT in ws and returns normally.
 * Used by tests to show that an expired wait is reported, not hung. */
MOE_EXPORT int moe_selftest_wait_timeout(const moe_config* cfg, int64_t timeout_ns,
                              void* ws, void* stream);

/* ---- dispatch without a workspace ------------------------------------------
 * No counterpart in the paper: an addition for callers that cannot allocate
 * device memory -- code running inside a host framework that owns every
 * device allocation and gives a plugin none of its own, or a latency-critical
 * caller that cannot afford the device-wide synchronisation of cudaMalloc.
 * Same outputs as moe_dispatch (same kernels, bit for bit) but no `ws`
 * argument: the dispatch scratch (token bitmaps and prefix counts,
 * 2 * P * ceil(T/32) * N_r 32-bit words with P = top_k under
 * MOE_PRIORITY_SLOT and 1 otherwise, each half rounded up to 256 bytes) comes
 * from a 2 MiB array in device memory that belongs to the library, so every
 * GPU that loads the library holds those 2 MiB until the process exits.
 * Shapes whose scratch exceeds 2 MiB return MOE_ERR_UNSUPPORTED before any
 * launch (e.g. T up to 32768 tokens at N_r = 256 with token priority; under
 * slot-major priority with top_k = 8 and N_r = 64, T up to 16384).  The call
 * allocates nothing.  The array used is the one of the calling thread's
 * current CUDA context (the current device's primary context unless the
 * caller made another context current), so `stream` must belong to that
 * context.  The first call in each context looks up the array's device
 * address there (cudaGetSymbolAddress) and keeps it for later calls; make
 * that first call before any stream capture.  Every call in a context shares
 * the one array and leaves its contents behind; the kernels rewrite all of it
 * before reading, so nothing needs clearing, but calls that overlap on the
 * GPU (other streams, other threads) race on it and must be serialised by
 * the caller.  Bad routing indices are dropped as in moe_dispatch; there is
 * no status word to report them, but their slot_row entries are -2.
 *   x, topk_idx, counts, kept, offsets, slot_row, row_slot, x_disp,
 *   x_disp_scales: as moe_dispatch. */
MOE_EXPORT int moe_dispatch_noalloc(const moe_config* cfg, const void* x, const int32_t* topk_idx,
                                    int32_t* counts, int32_t* kept, int32_t* offsets,
                                    int32_t* slot_row, int32_t* row_slot, void* x_disp,
                                    float* x_disp_scales, void* stream);

/* ---- backward of the layer (fp32 and bf16 layers) ------------------------
 * Gradients of J = sum_t <dout_t, out_t> + lam * L_balance with respect to x,
 * W_r, the per-expert logit bias and every routed and shared expert's
 * weights and biases.  The pages ("論文解説: DeepSeekMoE" §共有エキスパート機構,
 * §ルーティングとバランス損失, §アルゴリズム; "Sparse MoE Top-Kルーティング"
 * §解決策2) define the forward only; this is its derivative, read as:
 *   - the top-K choice, the capacity decisions and f_j (a fraction of counts)
 *     pass no gradient;
 *   - slot (t, k) gets a = <dout_t, y of the slot> if kept, <dout_t, x_t> if
 *     dropped with MOE_OVERFLOW_PASS, else 0; with S = sum over the selected
 *     s, ds of the slot's expert += (a_k - sum_k' a_k' g_k') / S; P_j adds
 *     lam * alpha * N_r * f_j / T to every ds_tj; dl = s * (ds - <s, ds>);
 *   - dW_r = dl^T x; dx gets dl W_r; with MOE_BIAS_LOGITS the bias gets
 *     sum_t dl, with MOE_BIAS_SELECTION (selection only) zero;
 *   - a kept slot's expert sees dy = g * dout_t, a shared expert dout_t;
 *     z = W1 x + b1 is recomputed; dz = (W2^T dy) * SiLU'(z); dW2 = dy SiLU(z)^T,
 *     dW1 = dz x^T, db1 / db2 the sums of dz / dy; dx gets W1^T dz of each
 *     kept slot, and g * dout_t of each slot dropped with pass-through.
 * MOE_FP8_E4M3_BLOCK returns MOE_ERR_UNSUPPORTED.  bf16 layers run every
 * expert GEMM (the recompute of z, dh, dx, dW1, dW2) on the tensor cores with
 * fp32 accumulation over bf16 copies of dy = g * dout, SiLU(z), SiLU'(z) and
 * dz; fp32 layers run fp32 arithmetic throughout.  Every reduction runs in a
 * fixed order (bit-reproducible).  Inputs are the forward's inputs and the
 * results of its stages on the same batch; outputs are fp32 and written in
 * full (experts no slot reached get zero gradients).  All pointers are device
 * memory, 16-byte aligned; NULL only where marked. */
typedef struct moe_backward_io {
    /* forward inputs */
    const void* x;              /* (T, d_model) activation dtype */
    const float* W_r;           /* (N_r, d_model) */
    const void* W1;             /* (N_r, d_ff, d_model) activation dtype */
    const float* b1;            /* (N_r, d_ff) */
    const void* W2;             /* (N_r, d_model, d_ff) */
    const float* b2;            /* (N_r, d_model) */
    const void* Ws1;            /* (n_shared, d_ff_shared, d_model); NULL if n_shared == 0 */
    const float* bs1;           /* (n_shared, d_ff_shared) */
    const void* Ws2;            /* (n_shared, d_model, d_ff_shared) */
    const float* bs2;           /* (n_shared, d_model) */
    /* results of the forward stages */
    const float* logits;        /* (T, N_r): moe_route's logits_out (the logits the softmax saw) */
    const int32_t* topk_idx;    /* (T, K) moe_route */
    const float* gates;         /* (T, K) moe_route */
    const int32_t* counts;      /* (N_r) moe_dispatch: pre-capacity counts */
    const int32_t* offsets;     /* (N_r + 1) moe_dispatch */
    const int32_t* slot_row;    /* (T, K) moe_dispatch */
    const int32_t* row_slot;    /* (R_cap) moe_dispatch */
    const void* x_disp;         /* (x_disp rows, d_model) moe_dispatch */
    const void* y;              /* (y rows, d_model) moe_expert_ffn */
    /* upstream gradient */
    const void* dout;           /* (T, d_model) activation dtype */
    /* gradients, fp32 */
    float* dx;                  /* (T, d_model) */
    float* dW_r;                /* (N_r, d_model) */
    float* d_logit_bias;        /* (N_r) or NULL */
    float* dW1;                 /* (N_r, d_ff, d_model) */
    float* db1;                 /* (N_r, d_ff) */
    float* dW2;                 /* (N_r, d_model, d_ff) */
    float* db2;                 /* (N_r, d_model) */
    float* dWs1;                /* (n_shared, d_ff_shared, d_model); NULL if n_shared == 0 */
    float* dbs1;                /* (n_shared, d_ff_shared) */
    float* dWs2;                /* (n_shared, d_model, d_ff_shared) */
    float* dbs2;                /* (n_shared, d_model) */
} moe_backward_io;

/* Bytes of the scratch moe_layer_backward needs (fp32 per-slot, per-token
 * and per-row intermediates).  FP8 layers: MOE_ERR_UNSUPPORTED. */
MOE_EXPORT int moe_backward_workspace_size(const moe_config* cfg, size_t* bytes);

/* Enqueues the backward on `stream`.  lam: weight of the balance loss in J
 * (finite).  bws: caller scratch of moe_backward_workspace_size() bytes,
 * 256-byte aligned, any contents (fully rewritten before it is read).  The
 * first 4 bytes of bws receive this call's device status word (0, or
 * MOE_DEV_TIMEOUT when a bounded wait of a tensor-core kernel gave up, the
 * gradients then being incomplete); moe_get_device_status(cfg, bws, ...)
 * reads it like a forward workspace's. */
MOE_EXPORT int moe_layer_backward(const moe_config* cfg, float lam, const moe_backward_io* io,
                                  void* bws, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */

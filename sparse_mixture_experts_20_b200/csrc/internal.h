// Internal (non-exported) launch interface between the C ABI layer and the
// kernel files.  Every launcher enqueues on `stream` and returns the
// cudaError_t of the launch.
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include "../../include/moe_b200.h"

namespace moe {

// Named NVTX range over one entry point (the enqueue of its kernels), for
// profiler timelines; without an attached tool the calls do nothing.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

// Workspace layout: byte offsets of every region, all 256-byte aligned.
struct WsLayout {
    size_t status;        // int32 status word (+ padding)
    size_t psum;          // (route_blocks, N_r) f32: per-block sums of s
    size_t bitmap;        // (T_words, N_r) u32: bit t%32 of word t/32 set if t selected j
    size_t word_base;     // (T_words, N_r) i32: slots of j in earlier words
    size_t h_r;           // routed hidden activations (R_cap, d_ff)
    size_t h_r_scales;    // FP8: (R_cap, d_ff/128) f32
    size_t h_s;           // shared hidden activations (n_shared*T, d_ff_shared)
    size_t h_s_scales;    // FP8: (n_shared*T, d_ff_shared/128) f32
    size_t router_w3;     // tensor-core router: (N_r, 3 d) bf16 planes of W_r
    size_t router_part;   // tensor-core router: (ksplit, T, N_r) f32 partial logits
    size_t router_logits; // tensor-core router: (T, N_r) f32 summed logits
    // used by moe_layer_forward only
    size_t x_disp;
    size_t x_disp_scales;
    size_t y;
    size_t topk_idx, gates, counts, kept, offsets, slot_row, row_slot;
    size_t total;
};

struct Dims {
    int T, d, E, K, dff, S, dffs;
    int capacity;   // -1: none
    int r_cap;
    int x_disp_rows;
    int y_rows;
    int dtype;
    int bias_mode;  // 0: logit_bias enters the logits; 1: only the top-K keys
    int slot_major; // capacity ranks: 0 token order, 1 slot-major
    int passthrough;// a slot over the capacity adds gate * x
    float alpha;
    int route_blocks;
    int t_words;
    int planes;     // token bitmaps per word: 1, or K (one per slot) when slot_major
};

constexpr int kRouteTokens = 32;    // tokens per router block

// Programmatic dependent launch is on unless the environment variable
// MOE_PDL is "0" (read once).
bool pdl_enabled();


int validate(const moe_config* cfg, Dims* dm);
WsLayout ws_layout(const Dims& dm);

// elements
inline size_t act_bytes(int dtype) { return dtype == MOE_F32 ? 4 : 2; }
inline size_t wt_bytes(int dtype) { return dtype == MOE_F32 ? 4 : (dtype == MOE_BF16 ? 2 : 1); }

// Scratch of the tensor-core router (workspace regions; unused otherwise).
struct RouterScratch {
    void* w3;
    float* part;
    float* logits;
    int32_t* status;
};

// Tile plan of the tensor-core router: m-tiles of 128 tokens, nt tiles of bn
// experts, ksplit splits of K = 3 d; pair: m-tiles two at a time on CTA pairs.
struct RouterTcPlan {
    int mt, nt, bn, ksplit, pair;
};

bool router_uses_small(const Dims& dm);
bool router_uses_tc(const Dims& dm);
RouterTcPlan router_tc_plan(const Dims& dm);
cudaError_t launch_router_tc(const Dims& dm, const RouterTcPlan& plan, const void* x, const float* W_r,
                             void* w3, float* part, int32_t* status, cudaStream_t st);

cudaError_t launch_router(const Dims& dm, const void* x, const float* W_r, const float* logit_bias,
                          int32_t* topk_idx, float* gates, float* logits_out, float* psum,
                          const RouterScratch& rs, cudaStream_t st);

// Balance statistics computed by the dispatch scan (moe_layer_forward): the
// router's per-block partial sums of s and the outputs; f == nullptr: none.
struct BalanceArgs {
    const float* psum;
    int blocks, T, K;
    float alpha;
    float* f;
    float* P;
    float* loss;
};

cudaError_t launch_dispatch(const Dims& dm, const void* x, const int32_t* topk_idx,
                            int32_t* counts, int32_t* kept, int32_t* offsets,
                            int32_t* slot_row, int32_t* row_slot, void* x_disp,
                            float* x_disp_scales, uint32_t* bitmap, int32_t* word_base,
                            int32_t* status, cudaStream_t st, const BalanceArgs* bal = nullptr);

cudaError_t launch_combine(const Dims& dm, const void* y, const float* gates,
                           const int32_t* slot_row, const void* x, void* out, cudaStream_t st);

cudaError_t launch_balance(const Dims& dm, const int32_t* counts, const float* psum,
                           float* f, float* P, float* loss, cudaStream_t st);

// One group of segments of a grouped GEMM C = act(A B^T + bias).
struct GemmGroup {
    const void* A;          // (a_rows, K) rows; element type per engine
    int a_rows;             // rows addressable through A (for the TMA map)
    int a_row_base;         // first A row of segment 0
    int a_seg_stride;       // A rows between consecutive fixed segments (shared group)
    const float* a_scales;  // FP8: (a_rows, K/128)
    const void* B;          // (n_mats, N, K)
    int n_mats;
    const float* b_scales;  // FP8: (n_mats, N/128, K/128)
    const float* bias;      // (n_mats, N)
    void* C;                // output rows
    int c_rows;
    int c_row_base;
    float* c_scales;        // FP8 GEMM1 output scales (c_rows, N/128)
    int N, K;
    // segments: routed groups take rows from offsets; fixed groups have
    // n_fixed segments of fixed_rows rows each.
    const int32_t* offsets; // (n_mats+1) or nullptr for a fixed group
    int fixed_rows;
    // routed group: segment i uses the weights, biases and scales of matrix
    // seg_mat[i] (device, n_mats entries) instead of matrix i, among n_weights
    // matrices (0: n_mats); nullptr: segment i is matrix i
    const int32_t* seg_mat;
    int n_weights;
};

struct GemmArgs {
    GemmGroup g[2];         // g[0] routed, g[1] shared (n_mats == 0 if none)
    int silu;               // 1: first layer (bias + SiLU), 0: second layer (bias)
    int out_fp8;            // FP8 engine: quantise the output (first layer)
    int32_t* status;
};

cudaError_t launch_grouped_ffn_f32(const Dims& dm, const GemmArgs& a, cudaStream_t st);
cudaError_t launch_grouped_ffn_bf16(const Dims& dm, const GemmArgs& a, cudaStream_t st);
cudaError_t launch_grouped_ffn_bf16_pair(const Dims& dm, const GemmArgs& a, cudaStream_t st);
// CTA-pair kernels are used unless the environment variable MOE_GEMM_PAIR is "0".
bool gemm_pairs_enabled();
cudaError_t launch_grouped_ffn_fp8(const Dims& dm, const GemmArgs& a, cudaStream_t st);

cudaError_t launch_wait_selftest(int64_t timeout_ns, int32_t* status, cudaStream_t st);

// TMA tensor maps (tma_host.cu).  `map` points at a CUtensorMap.
bool encode_tma_2d(void* map, const void* base, int rows, int K, int elem, int box_rows);
bool encode_tma_3d(void* map, const void* base, int n_mats, int N, int K, int elem, int box_rows);
bool encode_tma_2d_store64(void* map, const void* base, int rows, int cols, int elem, int box_rows);
int device_sm_count();

// Records a failed CUDA call for moe_last_cuda_error() on this thread.
void note_cuda_error(int err);

// Adds n to the process-wide kernel launch counter (moe_kernel_launches).
void count_launches(int n = 1);

// One group of a grouped GEMM of the backward (bwd_gemm.cu), bf16 operands.
// M-ragged kinds: C[rows of segment i, N] = A[rows, K] op(B_i); K-ragged
// (BWD_WGRAD): C_i[M, N] = A[K rows of i, M]^T B[K rows of i, N].
struct BwdGemmGroup {
    int n_mats;              // segments (matrices); 0: group unused
    const int32_t* seg;      // (n_mats + 1) device row offsets (16-row multiples apart), or nullptr
    int fixed;               // rows of every segment when seg is nullptr
    int M, N, K;             // M-ragged: N, K; K-ragged: M, N
    const void* A;           // (a_rows, a_cols) row-major
    int a_rows, a_cols;
    int a_row_base;          // first A row (K row when K-ragged) of segment 0
    int a_mat_stride;        // fixed segments: rows between segments
    const void* B;           // (b_mats, b_rows, b_cols) row-major
    int b_mats, b_rows, b_cols;
    int b_col_stride;        // K-ragged: B column offset of matrix i
    int b_z_mat;             // 1: B matrix index = segment index; 0: matrix 0
    const float* bias;       // recompute: (n_mats, N)
    const void* aux;         // dgrad-SiLU: SiLU'(z) bf16, addressed like out0
    void* out0;
    void* out1;              // recompute: SiLU'(z)
    int c_rows;              // M-ragged: rows of the output matrices (for their TMA store maps)
    int c_row_base;          // M-ragged: first output row of segment 0 (routed) or of all
    int c_mat_rows;          // fixed segments: output rows between segments
    int c_col_stride;        // M-ragged: output column offset of segment i
    int ldc;                 // output row stride (elements)
    long long c_mat_elems;   // K-ragged: elements between the matrices' outputs
    int out_bf16;            // BWD_DGRAD_F32: write bf16 instead of fp32
};

struct BwdGemmArgs {
    BwdGemmGroup g[2];       // routed, shared (n_mats == 0 if none)
    int32_t* status;
};

enum BwdGemmKind {
    BWD_RECOMPUTE = 0,       // M-ragged, B K-major; out0 = SiLU(v), out1 = SiLU'(v), v = acc + bias (bf16)
    BWD_DGRAD_SILU = 1,      // M-ragged, B MN-major; out0 = acc * aux (bf16)
    BWD_DGRAD_F32 = 2,       // M-ragged, B MN-major; out0 = acc (fp32, or bf16 with out_bf16)
    BWD_WGRAD = 3,           // K-ragged, A and B MN-major; out0 = acc (fp32), zeros for K = 0
};

cudaError_t launch_bwd_gemm(BwdGemmKind kind, const BwdGemmArgs& a, cudaStream_t st);

// Layer backward (backward.cu): scratch bytes and the launch sequence.
size_t backward_ws_bytes(const Dims& dm);
cudaError_t launch_backward(const Dims& dm, float lam, const moe_backward_io& io, void* bws,
                            cudaStream_t st);

// Launches `kernel` on `st` with programmatic stream serialization (the
// kernel must call pdl_wait() before it touches global memory) and, with
// cluster_x > 1, in clusters of cluster_x CTAs along x.  Returns the launch
// error; counts the launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       int cluster_x, Args&&... args) {
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    ++n;
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = static_cast<unsigned>(cluster_x);
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = n;
    count_launches(1);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe

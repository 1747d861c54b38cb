// C ABI of the MoE layer library: argument checks, workspace layout and the
// stage sequence.  Every entry point validates on the host before launching
// anything, and returns a MOE_* status; no C++ exception crosses the ABI.
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {
thread_local int g_last_cuda_error = 0;

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    g_last_cuda_error = static_cast<int>(e);
    return MOE_ERR_CUDA;
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// C = ceil(cf * T * K / N_r), exact on the fp32 value of cf; C >= T can
// never bind (an expert is chosen at most once per token) and is clamped to
// 2^30.
int capacity_of(float cf, int T, int K, int E) {
    if (!(cf > 0.f)) return -1;
    int e2 = 0;
    const float fr = std::frexp(cf, &e2);                 // cf = fr * 2^e2, fr in [0.5, 1)
    const long long mant = static_cast<long long>(std::ldexp(static_cast<double>(fr), 24));  // exact
    const int shift = e2 - 24;                           // cf = mant * 2^shift
    const __int128 num = static_cast<__int128>(mant) * T * K;
    __int128 c;
    if (shift >= 0) {
        if (shift > 40) return 1 << 30;
        const __int128 v = num << shift;
        c = (v + E - 1) / E;
    } else {
        if (-shift > 100) return 1;
        const __int128 den = static_cast<__int128>(E) << (-shift);
        c = (num + den - 1) / den;
    }
    if (c > (1 << 30)) return 1 << 30;
    return static_cast<int>(c);
}

}  // namespace

int validate(const moe_config* cfg, Dims* dm) {
    if (!cfg || !dm) return MOE_ERR_INVALID_ARG;
    const moe_config& c = *cfg;
    if (c.T < 1 || c.d_model < 1 || c.n_routed < 1 || c.top_k < 1 || c.d_ff < 1 || c.n_shared < 0)
        return MOE_ERR_INVALID_ARG;
    if (c.top_k > c.n_routed) return MOE_ERR_INVALID_ARG;
    if (c.n_shared > 0 && c.d_ff_shared < 1) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(c.capacity_factor) || c.capacity_factor < 0.f || !std::isfinite(c.alpha))
        return MOE_ERR_INVALID_ARG;
    if (c.dtype != MOE_F32 && c.dtype != MOE_BF16 && c.dtype != MOE_FP8_E4M3_BLOCK) return MOE_ERR_INVALID_ARG;
    if (c.bias_mode != MOE_BIAS_LOGITS && c.bias_mode != MOE_BIAS_SELECTION) return MOE_ERR_INVALID_ARG;
    if (c.capacity_priority != MOE_PRIORITY_TOKEN && c.capacity_priority != MOE_PRIORITY_SLOT) return MOE_ERR_INVALID_ARG;
    if (c.overflow_mode != MOE_OVERFLOW_DROP && c.overflow_mode != MOE_OVERFLOW_PASS) return MOE_ERR_INVALID_ARG;
    if (c.n_routed > 256 || c.top_k > 16 || c.n_shared > 8) return MOE_ERR_UNSUPPORTED;
    const int q = c.dtype == MOE_FP8_E4M3_BLOCK ? 128 : 64;
    if (c.d_model % q || c.d_ff % q || (c.n_shared > 0 && c.d_ff_shared % q)) return MOE_ERR_UNSUPPORTED;
    if (static_cast<long long>(c.T) * c.top_k > (1ll << 30)) return MOE_ERR_UNSUPPORTED;
    const long long big = static_cast<long long>(c.T) * (c.top_k + c.n_shared + 1);
    if (big > (1ll << 30)) return MOE_ERR_UNSUPPORTED;
    dm->T = c.T;
    dm->d = c.d_model;
    dm->E = c.n_routed;
    dm->K = c.top_k;
    dm->dff = c.d_ff;
    dm->S = c.n_shared;
    dm->dffs = c.n_shared > 0 ? c.d_ff_shared : 0;
    dm->dtype = c.dtype;
    dm->bias_mode = c.bias_mode;
    dm->slot_major = c.capacity_priority == MOE_PRIORITY_SLOT ? 1 : 0;
    dm->passthrough = c.overflow_mode == MOE_OVERFLOW_PASS ? 1 : 0;
    dm->alpha = c.alpha;
    dm->capacity = capacity_of(c.capacity_factor, c.T, c.top_k, c.n_routed);
    long long rcap = static_cast<long long>(c.T) * c.top_k;
    if (dm->capacity >= 0) {
        const long long lim = static_cast<long long>(c.n_routed) * dm->capacity;
        if (lim < rcap) rcap = lim;
    }
    dm->r_cap = static_cast<int>(rcap);
    dm->x_disp_rows = dm->r_cap + ((c.dtype == MOE_FP8_E4M3_BLOCK && c.n_shared > 0) ? c.T : 0);
    dm->y_rows = dm->r_cap + c.n_shared * c.T;
    dm->route_blocks = (c.T + kRouteTokens - 1) / kRouteTokens;
    dm->t_words = (c.T + 31) / 32;
    dm->planes = dm->slot_major ? c.top_k : 1;
    return MOE_OK;
}

WsLayout ws_layout(const Dims& dm) {
    WsLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t o = off; off = align256(off + bytes); return o; };
    const bool fp8 = dm.dtype == MOE_FP8_E4M3_BLOCK;
    const size_t hb = dm.dtype == MOE_F32 ? 4 : (dm.dtype == MOE_BF16 ? 2 : 1);
    L.status = take(256);
    L.psum = take(static_cast<size_t>(dm.route_blocks) * dm.E * 4);
    L.bitmap = take(static_cast<size_t>(dm.planes) * dm.t_words * dm.E * 4);
    L.word_base = take(static_cast<size_t>(dm.planes) * dm.t_words * dm.E * 4);
    L.h_r = take(static_cast<size_t>(dm.r_cap) * dm.dff * hb);
    L.h_r_scales = take(fp8 ? static_cast<size_t>(dm.r_cap) * (dm.dff / 128) * 4 : 0);
    L.h_s = take(static_cast<size_t>(dm.S) * dm.T * dm.dffs * hb);
    L.h_s_scales = take(fp8 ? static_cast<size_t>(dm.S) * dm.T * (dm.dffs / 128) * 4 : 0);
    if (router_uses_tc(dm)) {
        const RouterTcPlan rp = router_tc_plan(dm);
        L.router_w3 = take(static_cast<size_t>(dm.E) * 3 * dm.d * 2);
        L.router_part = take(static_cast<size_t>(rp.ksplit) * dm.T * dm.E * 4);
        L.router_logits = take(static_cast<size_t>(dm.T) * dm.E * 4);
    } else {
        L.router_w3 = L.router_part = L.router_logits = take(0);
    }
    L.x_disp = take(static_cast<size_t>(dm.x_disp_rows) * dm.d * hb);
    L.x_disp_scales = take(fp8 ? static_cast<size_t>(dm.x_disp_rows) * (dm.d / 128) * 4 : 0);
    L.y = take(static_cast<size_t>(dm.y_rows) * dm.d * (dm.dtype == MOE_F32 ? 4 : 2));
    L.topk_idx = take(static_cast<size_t>(dm.T) * dm.K * 4);
    L.gates = take(static_cast<size_t>(dm.T) * dm.K * 4);
    L.counts = take(static_cast<size_t>(dm.E) * 4);
    L.kept = take(static_cast<size_t>(dm.E) * 4);
    L.offsets = take(static_cast<size_t>(dm.E + 1) * 4);
    L.slot_row = take(static_cast<size_t>(dm.T) * dm.K * 4);
    L.row_slot = take(static_cast<size_t>(dm.r_cap) * 4);
    L.total = off;
    return L;
}

namespace {

template <typename T> T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

RouterScratch router_scratch(void* ws, const WsLayout& L) {
    RouterScratch rs;
    rs.w3 = at<uint8_t>(ws, L.router_w3);
    rs.part = at<float>(ws, L.router_part);
    rs.logits = at<float>(ws, L.router_logits);
    rs.status = at<int32_t>(ws, L.status);
    return rs;
}

// Builds the two grouped-GEMM launches of the expert FFN and runs them.
// seg_mat (device, n_seg entries) or nullptr: the routed group is n_seg
// caller-made segments over x_disp (offsets has n_seg + 1 entries), segment i
// computed with expert seg_mat[i] of the dm.E held.
int run_expert_ffn(const Dims& dm, const WsLayout& L, const void* x, const void* x_disp,
                   const float* x_disp_scales, const int32_t* offsets,
                   const void* W1, const float* W1_scales, const float* b1,
                   const void* W2, const float* W2_scales, const float* b2,
                   const void* Ws1, const float* Ws1_scales, const float* bs1,
                   const void* Ws2, const float* Ws2_scales, const float* bs2,
                   void* y, void* ws, cudaStream_t st, const int32_t* seg_mat = nullptr, int n_seg = 0) {
    const bool fp8 = dm.dtype == MOE_FP8_E4M3_BLOCK;
    void* h_r = at<uint8_t>(ws, L.h_r);
    void* h_s = at<uint8_t>(ws, L.h_s);
    float* h_r_sc = fp8 ? at<float>(ws, L.h_r_scales) : nullptr;
    float* h_s_sc = fp8 ? at<float>(ws, L.h_s_scales) : nullptr;
    int32_t* status = at<int32_t>(ws, L.status);

    GemmArgs g1{};
    g1.silu = 1;
    g1.out_fp8 = fp8 ? 1 : 0;
    g1.status = status;
    {
        GemmGroup& r = g1.g[0];
        r.A = x_disp; r.a_rows = dm.r_cap; r.a_row_base = 0; r.a_seg_stride = 0;
        r.a_scales = x_disp_scales;
        r.B = W1; r.n_mats = dm.E; r.b_scales = W1_scales; r.bias = b1;
        r.C = h_r; r.c_rows = dm.r_cap; r.c_row_base = 0; r.c_scales = h_r_sc;
        r.N = dm.dff; r.K = dm.d; r.offsets = offsets; r.fixed_rows = 0;
        if (seg_mat) { r.n_mats = n_seg; r.seg_mat = seg_mat; r.n_weights = dm.E; }
    }
    if (dm.S > 0) {
        GemmGroup& s = g1.g[1];
        if (fp8) { s.A = x_disp; s.a_rows = dm.x_disp_rows; s.a_row_base = dm.r_cap; s.a_scales = x_disp_scales; }
        else     { s.A = x;      s.a_rows = dm.T;           s.a_row_base = 0;        s.a_scales = nullptr; }
        s.a_seg_stride = 0;
        s.B = Ws1; s.n_mats = dm.S; s.b_scales = Ws1_scales; s.bias = bs1;
        s.C = h_s; s.c_rows = dm.S * dm.T; s.c_row_base = 0; s.c_scales = h_s_sc;
        s.N = dm.dffs; s.K = dm.d; s.offsets = nullptr; s.fixed_rows = dm.T;
    }
    GemmArgs g2{};
    g2.silu = 0;
    g2.out_fp8 = 0;
    g2.status = status;
    {
        GemmGroup& r = g2.g[0];
        r.A = h_r; r.a_rows = dm.r_cap; r.a_row_base = 0; r.a_seg_stride = 0; r.a_scales = h_r_sc;
        r.B = W2; r.n_mats = dm.E; r.b_scales = W2_scales; r.bias = b2;
        r.C = y; r.c_rows = dm.y_rows; r.c_row_base = 0; r.c_scales = nullptr;
        r.N = dm.d; r.K = dm.dff; r.offsets = offsets; r.fixed_rows = 0;
        if (seg_mat) { r.n_mats = n_seg; r.seg_mat = seg_mat; r.n_weights = dm.E; }
    }
    if (dm.S > 0) {
        GemmGroup& s = g2.g[1];
        s.A = h_s; s.a_rows = dm.S * dm.T; s.a_row_base = 0; s.a_seg_stride = dm.T; s.a_scales = h_s_sc;
        s.B = Ws2; s.n_mats = dm.S; s.b_scales = Ws2_scales; s.bias = bs2;
        s.C = y; s.c_rows = dm.y_rows; s.c_row_base = dm.r_cap; s.c_scales = nullptr;
        s.N = dm.d; s.K = dm.dffs; s.offsets = nullptr; s.fixed_rows = dm.T;
    }
    cudaError_t e;
    if (dm.dtype == MOE_F32) {
        e = launch_grouped_ffn_f32(dm, g1, st);
        if (e == cudaSuccess) e = launch_grouped_ffn_f32(dm, g2, st);
    } else if (dm.dtype == MOE_BF16) {
        if (gemm_pairs_enabled()) {
            e = launch_grouped_ffn_bf16_pair(dm, g1, st);
            if (e == cudaSuccess) e = launch_grouped_ffn_bf16_pair(dm, g2, st);
        } else {
            e = launch_grouped_ffn_bf16(dm, g1, st);
            if (e == cudaSuccess) e = launch_grouped_ffn_bf16(dm, g2, st);
        }
    } else {
        e = launch_grouped_ffn_fp8(dm, g1, st);
        if (e == cudaSuccess) e = launch_grouped_ffn_fp8(dm, g2, st);
    }
    return cuda_status(e);
}

bool ffn_args_ok(const Dims& dm, const void* x, const void* x_disp, const float* x_disp_scales,
                 const int32_t* offsets, const void* W1, const float* W1_scales, const float* b1,
                 const void* W2, const float* W2_scales, const float* b2, const void* Ws1,
                 const float* Ws1_scales, const float* bs1, const void* Ws2, const float* Ws2_scales,
                 const float* bs2) {
    const bool fp8 = dm.dtype == MOE_FP8_E4M3_BLOCK;
    const void* need[] = {x_disp, offsets, W1, b1, W2, b2};
    for (const void* p : need) if (!p || !aligned16(p)) return false;
    if (fp8 && (!x_disp_scales || !W1_scales || !W2_scales)) return false;
    if (dm.S > 0) {
        const void* sh[] = {Ws1, bs1, Ws2, bs2};
        for (const void* p : sh) if (!p || !aligned16(p)) return false;
        if (fp8 && (!Ws1_scales || !Ws2_scales)) return false;
        if (!fp8 && (!x || !aligned16(x))) return false;
    }
    return true;
}

__global__ void wait_selftest_kernel(int64_t timeout_ns, int32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    volatile int* af = &abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        *af = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // nothing ever arrives on `bar`: the wait must give up and report
        mbar_wait_bounded(&bar, 0, af, status, static_cast<uint64_t>(timeout_ns));
    }
    __syncthreads();
}

}  // namespace

void note_cuda_error(int err) { g_last_cuda_error = err; }

bool pdl_enabled() {
    static const bool on = [] {
        const char* v = std::getenv("MOE_PDL");
        return !(v && v[0] == '0');
    }();
    return on;
}

static std::atomic<uint64_t> g_kernel_launches{0};
void count_launches(int n) { g_kernel_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

cudaError_t launch_wait_selftest(int64_t timeout_ns, int32_t* status, cudaStream_t st) {
    wait_selftest_kernel<<<1, 32, 0, st>>>(timeout_ns, status);
    count_launches();
    return cudaGetLastError();
}

}  // namespace moe

using namespace moe;

extern "C" {

int moe_workspace_size(const moe_config* cfg, size_t* bytes) {
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    *bytes = ws_layout(dm).total;
    return MOE_OK;
}

int moe_buffer_rows(const moe_config* cfg, int32_t* capacity, int32_t* r_cap,
                    int32_t* x_disp_rows, int32_t* y_rows) {
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (capacity) *capacity = dm.capacity;
    if (r_cap) *r_cap = dm.r_cap;
    if (x_disp_rows) *x_disp_rows = dm.x_disp_rows;
    if (y_rows) *y_rows = dm.y_rows;
    return MOE_OK;
}

int moe_workspace_init(const moe_config* cfg, void* ws, void* stream) {
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, ws_layout(dm).total, static_cast<cudaStream_t>(stream)));
}

int moe_get_device_status(const moe_config* cfg, void* ws, void* stream, int32_t* status, int32_t clear) {
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!ws || !status) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* dev = at<int32_t>(ws, ws_layout(dm).status);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemcpy(status, dev, sizeof(int32_t), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && clear) {
        e = cudaMemsetAsync(dev, 0, sizeof(int32_t), st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    return cuda_status(e);
}

int moe_last_cuda_error(void) { return g_last_cuda_error; }

uint64_t moe_kernel_launches(void) { return moe::g_kernel_launches.load(std::memory_order_relaxed); }

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_BAD_ROUTING: return "MOE_ERR_BAD_ROUTING";
        case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
        default: return "MOE_ERR_UNKNOWN";
    }
}

int moe_route(const moe_config* cfg, const void* x, const float* W_r, const float* logit_bias,
              int32_t* topk_idx, float* gates, float* logits_out, void* ws, void* stream) {
    NvtxRange nvtx("moe_route");
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!x || !W_r || !topk_idx || !gates || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W_r) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(dm);
    return cuda_status(launch_router(dm, x, W_r, logit_bias, topk_idx, gates, logits_out,
                                     at<float>(ws, L.psum), router_scratch(ws, L), static_cast<cudaStream_t>(stream)));
}

int moe_dispatch(const moe_config* cfg, const void* x, const int32_t* topk_idx, int32_t* counts,
                 int32_t* kept, int32_t* offsets, int32_t* slot_row, int32_t* row_slot, void* x_disp,
                 float* x_disp_scales, void* ws, void* stream) {
    NvtxRange nvtx("moe_dispatch");
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!x || !topk_idx || !counts || !kept || !offsets || !slot_row || !row_slot || !x_disp || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_disp) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_INVALID_ARG;
    if (dm.dtype == MOE_FP8_E4M3_BLOCK && !x_disp_scales) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(dm);
    return cuda_status(launch_dispatch(dm, x, topk_idx, counts, kept, offsets, slot_row, row_slot, x_disp,
                                       x_disp_scales, at<uint32_t>(ws, L.bitmap), at<int32_t>(ws, L.word_base),
                                       at<int32_t>(ws, L.status), static_cast<cudaStream_t>(stream)));
}

int moe_expert_ffn(const moe_config* cfg, const void* x, const void* x_disp, const float* x_disp_scales,
                   const int32_t* offsets, const void* W1, const float* W1_scales, const float* b1,
                   const void* W2, const float* W2_scales, const float* b2, const void* Ws1,
                   const float* Ws1_scales, const float* bs1, const void* Ws2, const float* Ws2_scales,
                   const float* bs2, void* y, void* ws, void* stream) {
    NvtxRange nvtx("moe_expert_ffn");
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!y || !ws || !aligned16(y) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_INVALID_ARG;
    if (!ffn_args_ok(dm, x, x_disp, x_disp_scales, offsets, W1, W1_scales, b1, W2, W2_scales, b2, Ws1,
                     Ws1_scales, bs1, Ws2, Ws2_scales, bs2))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(dm);
    return run_expert_ffn(dm, L, x, x_disp, x_disp_scales, offsets, W1, W1_scales, b1, W2, W2_scales, b2,
                          Ws1, Ws1_scales, bs1, Ws2, Ws2_scales, bs2, y, ws, static_cast<cudaStream_t>(stream));
}

int moe_expert_ffn_segments(const moe_config* cfg, const void* x_rows, const float* x_rows_scales,
                            const int32_t* seg_offsets, const int32_t* seg_expert, int32_t n_seg,
                            const void* W1, const float* W1_scales, const float* b1, const void* W2,
                            const float* W2_scales, const float* b2, void* y, void* ws, void* stream) {
    NvtxRange nvtx("moe_expert_ffn_segments");
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (dm.S != 0 || dm.K != 1 || dm.capacity >= 0) return MOE_ERR_INVALID_ARG;
    if (n_seg < 1 || n_seg > 256) return MOE_ERR_INVALID_ARG;
    if (!seg_expert || !aligned16(seg_expert)) return MOE_ERR_INVALID_ARG;
    if (!y || !ws || !aligned16(y) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_INVALID_ARG;
    if (!ffn_args_ok(dm, nullptr, x_rows, x_rows_scales, seg_offsets, W1, W1_scales, b1, W2, W2_scales, b2,
                     nullptr, nullptr, nullptr, nullptr, nullptr, nullptr))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(dm);
    return run_expert_ffn(dm, L, nullptr, x_rows, x_rows_scales, seg_offsets, W1, W1_scales, b1, W2, W2_scales,
                          b2, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, y, ws,
                          static_cast<cudaStream_t>(stream), seg_expert, n_seg);
}

int moe_combine(const moe_config* cfg, const void* y, const float* gates, const int32_t* slot_row,
                const void* x, void* out, void* stream) {
    NvtxRange nvtx("moe_combine");
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!y || !gates || !slot_row || !out || !aligned16(y) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if (dm.passthrough && (!x || !aligned16(x))) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_combine(dm, y, gates, slot_row, x, out, static_cast<cudaStream_t>(stream)));
}

int moe_balance_stats(const moe_config* cfg, const int32_t* counts, const void* ws, float* f, float* P,
                      float* loss, void* stream) {
    NvtxRange nvtx("moe_balance_stats");
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!counts || !ws || !f || !P || !loss) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(dm);
    const float* psum = reinterpret_cast<const float*>(static_cast<const uint8_t*>(ws) + L.psum);
    return cuda_status(launch_balance(dm, counts, psum, f, P, loss, static_cast<cudaStream_t>(stream)));
}

int moe_layer_forward(const moe_config* cfg, const void* x, const float* W_r, const float* logit_bias,
                      const void* W1, const float* W1_scales, const float* b1,
                      const void* W2, const float* W2_scales, const float* b2,
                      const void* Ws1, const float* Ws1_scales, const float* bs1,
                      const void* Ws2, const float* Ws2_scales, const float* bs2,
                      void* out, float* f, float* P, float* loss,
                      int32_t* topk_idx, float* gates, int32_t* counts, void* ws, void* stream) {
    NvtxRange nvtx("moe_layer_forward");
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!x || !W_r || !out || !f || !P || !loss || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W_r) || !aligned16(out) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(dm);
    const bool fp8 = dm.dtype == MOE_FP8_E4M3_BLOCK;
    int32_t* idx = topk_idx ? topk_idx : at<int32_t>(ws, L.topk_idx);
    float* g = gates ? gates : at<float>(ws, L.gates);
    int32_t* cnt = counts ? counts : at<int32_t>(ws, L.counts);
    void* x_disp = at<uint8_t>(ws, L.x_disp);
    float* x_disp_sc = fp8 ? at<float>(ws, L.x_disp_scales) : nullptr;
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* slot_row = at<int32_t>(ws, L.slot_row);
    void* y = at<uint8_t>(ws, L.y);
    if (!ffn_args_ok(dm, x, x_disp, x_disp_sc, offsets, W1, W1_scales, b1, W2, W2_scales, b2, Ws1,
                     Ws1_scales, bs1, Ws2, Ws2_scales, bs2))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_router(dm, x, W_r, logit_bias, idx, g, nullptr, at<float>(ws, L.psum),
                                  router_scratch(ws, L), st);
    if (e != cudaSuccess) return cuda_status(e);
    // the balance statistics come out of the dispatch scan (same arithmetic
    // as moe_balance_stats, one kernel fewer)
    const BalanceArgs bal{at<float>(ws, L.psum), dm.route_blocks, dm.T, dm.K, dm.alpha, f, P, loss};
    e = launch_dispatch(dm, x, idx, cnt, at<int32_t>(ws, L.kept), offsets, slot_row, at<int32_t>(ws, L.row_slot),
                        x_disp, x_disp_sc, at<uint32_t>(ws, L.bitmap), at<int32_t>(ws, L.word_base),
                        at<int32_t>(ws, L.status), st, &bal);
    if (e != cudaSuccess) return cuda_status(e);
    const int r = run_expert_ffn(dm, L, x, x_disp, x_disp_sc, offsets, W1, W1_scales, b1, W2, W2_scales, b2,
                                 Ws1, Ws1_scales, bs1, Ws2, Ws2_scales, bs2, y, ws, st);
    if (r != MOE_OK) return r;
    return cuda_status(launch_combine(dm, y, g, slot_row, x, out, st));
}

int moe_backward_workspace_size(const moe_config* cfg, size_t* bytes) {
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    if (dm.dtype == MOE_FP8_E4M3_BLOCK) return MOE_ERR_UNSUPPORTED;
    *bytes = backward_ws_bytes(dm);
    return MOE_OK;
}

int moe_layer_backward(const moe_config* cfg, float lam, const moe_backward_io* io, void* bws, void* stream) {
    NvtxRange nvtx("moe_layer_backward");
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (dm.dtype == MOE_FP8_E4M3_BLOCK) return MOE_ERR_UNSUPPORTED;
    if (!io || !bws || (reinterpret_cast<uintptr_t>(bws) & 255u) || !std::isfinite(lam)) return MOE_ERR_INVALID_ARG;
    const void* need[] = {io->x, io->W_r, io->W1, io->b1, io->W2, io->b2, io->logits, io->topk_idx, io->gates,
                          io->counts, io->offsets, io->slot_row, io->row_slot, io->x_disp, io->y, io->dout,
                          io->dx, io->dW_r, io->dW1, io->db1, io->dW2, io->db2};
    for (const void* p : need) if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
    if (io->d_logit_bias && !aligned16(io->d_logit_bias)) return MOE_ERR_INVALID_ARG;
    if (dm.S > 0) {
        const void* sh[] = {io->Ws1, io->bs1, io->Ws2, io->bs2, io->dWs1, io->dbs1, io->dWs2, io->dbs2};
        for (const void* p : sh) if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
    }
    return cuda_status(launch_backward(dm, lam, *io, bws, static_cast<cudaStream_t>(stream)));
}

int moe_selftest_wait_timeout(const moe_config* cfg, int64_t timeout_ns, void* ws, void* stream) {
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (timeout_ns < 1000) timeout_ns = 1000;
    if (timeout_ns > 10000000000ll) timeout_ns = 10000000000ll;
    const WsLayout L = ws_layout(dm);
    return cuda_status(launch_wait_selftest(timeout_ns, at<int32_t>(ws, L.status), static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

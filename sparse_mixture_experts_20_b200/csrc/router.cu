// Router: logits, softmax, top-K and gate renormalisation.
//
// "論文解説: DeepSeekMoE" §ルーティングとバランス損失: s_j = softmax(W_r x)_j,
// g_j = s_j / sum_{k in TopK} s_k; §アルゴリズム: the router is a Linear
// layer without bias.  "Sparse MoE Top-Kルーティング" §ルーティングの仕組み.
//
// The logits come from one of three producers, chosen by shape:
//   * router_small_kernel (N_r <= 32 and W_r fits in shared memory): W_r is
//     staged once per block by bulk asynchronous copies (one per expert row,
//     completed on an mbarrier); each warp takes 4 (or 2) tokens and one half
//     of the model dimension (16 warps), lanes split it with 16-byte loads of
//     x, a reduce-scatter over the lanes leaves each lane with whole partial
//     dot products, and the two halves are added in a fixed order.  x is read
//     once.
//   * the tensor-core router (router_tc.cu, bf16 x, larger N_r): W_r split into
//     three bf16 planes, one tcgen05 GEMM with K = 3 d, partial logits per K
//     split summed in split order by router_select_kernel as it loads them
//     (up to 4 splits) or first by router_reduce_kernel;
//   * router_generic_kernel (fp32 x with a large W_r): a shared-memory tiled
//     fp32 GEMM.
// All three end in select_block: per token a warp-wide softmax, a K-round
// arg-max (ties to the lower expert index) and the gates; per block the
// column sums of s over its 32 tokens go to psum in token order, so the
// balance statistics are bit-reproducible.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int TT = kRouteTokens;   // tokens per block
constexpr int KC = 32;             // columns per shared-memory chunk (generic kernel)
constexpr int NTHREADS = 256;
constexpr int kSelectSplits = 4;  // K splits the select kernel sums itself

template <typename XT> __device__ __forceinline__ float to_f(XT v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Order-preserving map of a float to an unsigned key: a > b as floats iff
// key(a) > key(b), with -0 folded onto +0 so that the two compare equal; every
// non-NaN value maps above 0, which stays free to mean "not selectable".
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// lg: TT rows of EPT*32 (+1 pad) softmax logits (any logit bias already
// added) and -inf in padded expert columns.  Rows of tokens >= T are ignored.
// Overwrites lg with s.  sel_bias (or nullptr): a per-expert bias that enters
// only the top-K keys (auxiliary-loss-free balancing, "Sparse MoE Top-K
// ルーティング" §解決策3); softmax, gates and the partial sums of s stay on lg.
template <int EPT, int NW = NTHREADS / 32>       // NW: warps of the calling block
__device__ __forceinline__ void select_block(float* lg_raw, int t0, int T, int E, int K,
                                             int32_t* __restrict__ topk_idx, float* __restrict__ gates,
                                             float* __restrict__ logits_out, float* __restrict__ psum,
                                             const float* __restrict__ sel_bias) {
    constexpr int NP = EPT * 32;
    float (*lg)[NP + 1] = reinterpret_cast<float (*)[NP + 1]>(lg_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll 1
    for (int i = 0; i < TT / NW; ++i) {
        const int r = warp + NW * i;
        const int t = t0 + r;
        if (t >= T) {                                 // zero s so psum ignores it
#pragma unroll
            for (int b = 0; b < EPT; ++b) lg[r][lane + 32 * b] = 0.f;
            continue;
        }
        float v[EPT];
#pragma unroll
        for (int b = 0; b < EPT; ++b) v[b] = lg[r][lane + 32 * b];
        if (logits_out) {
#pragma unroll
            for (int b = 0; b < EPT; ++b)
                if (lane + 32 * b < E) logits_out[static_cast<size_t>(t) * E + lane + 32 * b] = v[b];
        }
        // selection keys: the logits, plus the selection-only bias if any,
        // mapped to unsigned integers in the same order (0 = not selectable)
        uint32_t key[EPT];
#pragma unroll
        for (int b = 0; b < EPT; ++b) {
            const int j = lane + 32 * b;
            const float kv = (sel_bias != nullptr && j < E) ? v[b] + __ldg(sel_bias + j) : v[b];
            key[b] = j < E ? order_key(kv) : 0u;
        }
        uint32_t taken = 0;
        float vmax = 0.f, sel_v = 0.f;
        int sel_j = 0;
        for (int k = 0; k < K; ++k) {
            // this lane's largest free key, the lowest index among equals
            uint32_t bk = 0u;
            int bj = 0x7fffffff;
#pragma unroll
            for (int b = 0; b < EPT; ++b)
                if (!((taken >> b) & 1u) && key[b] > bk) { bk = key[b]; bj = lane + 32 * b; }
            // the warp's largest key, then the lowest index holding it
            const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
            bj = __reduce_min_sync(0xffffffffu, bk == wk ? bj : 0x7fffffff);
            float bv = order_key_value(wk);
            if (sel_bias != nullptr) {
                // the winner's softmax logit (its key includes the bias)
                float ub = v[0];
#pragma unroll
                for (int b = 1; b < EPT; ++b)
                    if (b == (bj >> 5)) ub = v[b];
                bv = __shfl_sync(0xffffffffu, ub, bj & 31);
            }
            if (k == 0) vmax = bv;
            if ((bj & 31) == lane) taken |= 1u << (bj >> 5);
            if (lane == k) { sel_v = bv; sel_j = bj; }
        }
        if (sel_bias != nullptr) {                    // the softmax maximum over all experts
            uint32_t m = 0u;
#pragma unroll
            for (int b = 0; b < EPT; ++b)
                if (lane + 32 * b < E) m = max(m, order_key(v[b]));
            vmax = order_key_value(__reduce_max_sync(0xffffffffu, m));
        }
        float e_sum = 0.f;
#pragma unroll
        for (int b = 0; b < EPT; ++b) {
            const float e = (lane + 32 * b < E) ? expf(v[b] - vmax) : 0.f;
            v[b] = e;
            e_sum += e;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) e_sum += __shfl_xor_sync(0xffffffffu, e_sum, off);
        const float inv = 1.0f / e_sum;
#pragma unroll
        for (int b = 0; b < EPT; ++b) lg[r][lane + 32 * b] = v[b] * inv;
        const float es = (lane < K) ? expf(sel_v - vmax) * inv : 0.f;
        float g_sum = es;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) g_sum += __shfl_xor_sync(0xffffffffu, g_sum, off);
        if (lane < K) {
            topk_idx[static_cast<size_t>(t) * K + lane] = sel_j;
            gates[static_cast<size_t>(t) * K + lane] = es / g_sum;
        }
    }
    __syncthreads();
    for (int j = tid; j < E; j += NW * 32) {
        float s = 0.f;
        for (int r = 0; r < TT; ++r) s += lg[r][j];
        psum[static_cast<size_t>(blockIdx.x) * E + j] = s;
    }
}

// ---------------------------------------------------------------- generic (fp32 x)

template <typename XT, int EPT>
__global__ void __launch_bounds__(NTHREADS)
router_generic_kernel(const XT* __restrict__ x, const float* __restrict__ W_r,
                      const float* __restrict__ logit_bias, int T, int d, int E, int K,
                      int32_t* __restrict__ topk_idx, float* __restrict__ gates,
                      float* __restrict__ logits_out, float* __restrict__ psum,
                      const float* __restrict__ sel_bias) {
    constexpr int NP = EPT * 32;
    __shared__ float xs[TT][KC + 1];
    __shared__ float wsh[(NP * (KC + 1) > TT * (NP + 1)) ? NP * (KC + 1) : TT * (NP + 1)];
    float (*wtile)[KC + 1] = reinterpret_cast<float (*)[KC + 1]>(wsh);
    float (*lg)[NP + 1] = reinterpret_cast<float (*)[NP + 1]>(wsh);
    pdl_wait();
    pdl_allow_next();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * TT;
    float acc[4][EPT];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < EPT; ++b) acc[a][b] = 0.f;
    for (int k0 = 0; k0 < d; k0 += KC) {
#pragma unroll
        for (int i = 0; i < (TT * KC) / NTHREADS; ++i) {
            const int e = tid + i * NTHREADS;
            const int r = e / KC, c = e % KC;
            const int t = t0 + r;
            xs[r][c] = (t < T) ? to_f<XT>(x[static_cast<size_t>(t) * d + k0 + c]) : 0.f;
        }
        for (int e = tid; e < NP * (KC / 4); e += NTHREADS) {
            const int r = e / (KC / 4), c4 = e % (KC / 4);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < E) v = *reinterpret_cast<const float4*>(W_r + static_cast<size_t>(r) * d + k0 + c4 * 4);
            wtile[r][c4 * 4 + 0] = v.x;
            wtile[r][c4 * 4 + 1] = v.y;
            wtile[r][c4 * 4 + 2] = v.z;
            wtile[r][c4 * 4 + 3] = v.w;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < KC; ++kk) {
            float xv[4], wv[EPT];
#pragma unroll
            for (int a = 0; a < 4; ++a) xv[a] = xs[warp * 4 + a][kk];
#pragma unroll
            for (int b = 0; b < EPT; ++b) wv[b] = wtile[lane + 32 * b][kk];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < EPT; ++b) acc[a][b] = fmaf(xv[a], wv[b], acc[a][b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < EPT; ++b) {
            const int j = lane + 32 * b;
            float v = -INFINITY;
            if (j < E) v = acc[a][b] + (logit_bias ? logit_bias[j] : 0.f);
            lg[warp * 4 + a][j] = v;
        }
    __syncthreads();
    select_block<EPT>(wsh, t0, T, E, K, topk_idx, gates, logits_out, psum, sel_bias);
}

// ---------------------------------------------------------------- small N_r

// After the call, v[i] of lane l holds the warp-wide sum of original index
// l * (N / 32) + i, for i < N / 32 (a reduce-scatter in 5 shuffle rounds).
template <int N>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[N], int lane) {
    static_assert(N >= 32 && (N & (N - 1)) == 0, "power of two >= 32");
#pragma unroll
    for (int s = 0; s < 5; ++s) {
        const int o = 16 >> s;
        const int half = (N >> s) / 2;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

constexpr uint64_t kStageWaitNs = 2000000000ull;

// Warps of the small router: two groups of 8 (one per half of the model
// dimension) when a warp's register tile is 32 accumulators, else one group.
template <int NE, int RT> struct SmallCfg {
    static constexpr int GROUPS = (RT * NE == 32) ? 2 : 1;
    static constexpr int WARPS = 8 * GROUPS;
};

template <typename XT, int NE, int RT>
__global__ void __launch_bounds__(SmallCfg<NE, RT>::WARPS * 32)
router_small_kernel(const XT* __restrict__ x, const float* __restrict__ W_r,
                    const float* __restrict__ logit_bias, int T, int d, int E, int K,
                    int32_t* __restrict__ topk_idx, float* __restrict__ gates,
                    float* __restrict__ logits_out, float* __restrict__ psum, int32_t* status,
                    const float* __restrict__ sel_bias) {
    extern __shared__ float4 wsm4[];                  // (NE, d) fp32, rows >= E zero
    float* wsm = reinterpret_cast<float*>(wsm4);
    __shared__ float lg[TT][32 + 1];
    __shared__ float lgp[2][TT][32 + 1];              // partial logits of the two halves of d
    __shared__ __align__(8) uint64_t wbar;
    __shared__ int abort_s;
    constexpr int GROUPS = SmallCfg<NE, RT>::GROUPS;
    constexpr int NT = SmallCfg<NE, RT>::WARPS * 32;
    constexpr int VEC = sizeof(XT) == 2 ? 8 : 4;      // elements per 16-byte load
    constexpr int NV = RT * NE;
    static_assert(NV == 32 || NV == 64, "register tile");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * TT;
    pdl_wait();
    pdl_allow_next();

    if (tid == 0) {
        abort_s = 0;
        mbar_init(&wbar, 1);
        fence_mbar_init();
        // rows 0..E-1 of W_r, d * 4 bytes each, land asynchronously
        mbar_arrive_expect_tx(&wbar, static_cast<uint32_t>(E) * d * 4);
        for (int e = 0; e < E; ++e)
            bulk_copy_g2s(wsm + static_cast<size_t>(e) * d, W_r + static_cast<size_t>(e) * d,
                          static_cast<uint32_t>(d) * 4, &wbar);
    }
    for (int i = E * d / 4 + tid; i < NE * d / 4; i += NT) wsm4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = tid; i < TT * 32; i += NT)
        if ((i & 31) >= NE) lg[i >> 5][i & 31] = -INFINITY;
    __syncthreads();
    if (!mbar_wait_bounded(&wbar, 0, &abort_s, status, kStageWaitNs)) {
        // the copies never completed (reported in the status word): leave the
        // outputs of this block unwritten rather than compute on garbage
        return;
    }

    // with two groups, warps 0..7 take columns [0, d/2) of every token and
    // warps 8..15 the rest
    const int half = warp >> 3, wg = warp & 7;
    const int k_begin = GROUPS == 2 ? half * (d / 2) : 0;
    const int k_end = (GROUPS == 2 && half == 0) ? d / 2 : d;
#pragma unroll 1
    for (int g = wg; g < TT / RT; g += 8) {
        float acc[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) acc[i] = 0.f;
        const XT* xr[RT];
        bool ok[RT];
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const int t = t0 + g * RT + r;
            ok[r] = t < T;
            xr[r] = x + static_cast<size_t>(ok[r] ? t : 0) * d;
        }
#pragma unroll 4
        for (int k = k_begin + lane * VEC; k < k_end; k += 32 * VEC) {
            float xv[RT][VEC];
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                const uint4 raw = ok[r] ? __ldg(reinterpret_cast<const uint4*>(xr[r] + k)) : make_uint4(0, 0, 0, 0);
                if (VEC == 8) {
                    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 f = __bfloat1622float2(h2[q]);
                        xv[r][2 * q] = f.x;
                        xv[r][2 * q + 1] = f.y;
                    }
                } else {
                    const float* f = reinterpret_cast<const float*>(&raw);
#pragma unroll
                    for (int q = 0; q < VEC; ++q) xv[r][q] = f[q];
                }
            }
#pragma unroll
            for (int e = 0; e < NE; ++e) {
                float w[VEC];
#pragma unroll
                for (int q = 0; q < VEC / 4; ++q) {
                    const float4 w4 = *reinterpret_cast<const float4*>(wsm + static_cast<size_t>(e) * d + k + 4 * q);
                    w[4 * q] = w4.x; w[4 * q + 1] = w4.y; w[4 * q + 2] = w4.z; w[4 * q + 3] = w4.w;
                }
#pragma unroll
                for (int r = 0; r < RT; ++r)
#pragma unroll
                    for (int q = 0; q < VEC; ++q) acc[r * NE + e] = fmaf(xv[r][q], w[q], acc[r * NE + e]);
            }
        }
        warp_reduce_scatter<NV>(acc, lane);
#pragma unroll
        for (int i = 0; i < NV / 32; ++i) {
            const int vi = lane * (NV / 32) + i;
            lgp[half][g * RT + vi / NE][vi % NE] = acc[i];
        }
    }
    __syncthreads();
    for (int i = tid; i < TT * NE; i += NT) {         // the two halves, in a fixed order
        const int r = i / NE, e = i % NE;
        const float l = GROUPS == 2 ? lgp[0][r][e] + lgp[1][r][e] : lgp[0][r][e];
        lg[r][e] = (e < E) ? l + (logit_bias ? logit_bias[e] : 0.f) : -INFINITY;
    }
    __syncthreads();
    select_block<1, SmallCfg<NE, RT>::WARPS>(&lg[0][0], t0, T, E, K, topk_idx, gates, logits_out, psum, sel_bias);
}

// ---------------------------------------------------------------- from precomputed logits

// One warp per token (32 warps: the block's 32 tokens at once).  The logits
// are the sum of the ks partial planes part[s][t][j] in split order; the
// loads of one split are all issued before any of them is used.
constexpr int SEL_THREADS = 1024;
static_assert(TT == SEL_THREADS / 32, "one warp per token");

template <int EPT>
__global__ void __launch_bounds__(SEL_THREADS)
router_select_kernel(const float* __restrict__ part, int ks, const float* __restrict__ logit_bias,
                     int T, int E, int K, int32_t* __restrict__ topk_idx, float* __restrict__ gates,
                     float* __restrict__ logits_out, float* __restrict__ psum,
                     const float* __restrict__ sel_bias) {
    constexpr int NP = EPT * 32;
    constexpr int PER = TT * NP / SEL_THREADS;
    __shared__ float lg[TT * (NP + 1)];
    pdl_wait();
    pdl_allow_next();
    const int t0 = blockIdx.x * TT;
    const size_t plane = static_cast<size_t>(T) * E;
    float acc[PER];
    bool ok[PER];
    const float* src[PER];
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        const int i = threadIdx.x + q * SEL_THREADS;
        const int r = i / NP, j = i % NP;
        const int t = t0 + r;
        ok[q] = j < E && t < T;
        src[q] = part + (ok[q] ? static_cast<size_t>(t) * E + j : 0);
        acc[q] = ok[q] ? __ldg(src[q]) : 0.f;
    }
    for (int sp = 1; sp < ks; ++sp) {
        float nx[PER];
#pragma unroll
        for (int q = 0; q < PER; ++q) nx[q] = ok[q] ? __ldg(src[q] + sp * plane) : 0.f;
#pragma unroll
        for (int q = 0; q < PER; ++q) acc[q] += nx[q];
    }
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        const int i = threadIdx.x + q * SEL_THREADS;
        const int r = i / NP, j = i % NP;
        lg[r * (NP + 1) + j] = ok[q] ? acc[q] + (logit_bias ? __ldg(logit_bias + j) : 0.f) : -INFINITY;
    }
    __syncthreads();
    select_block<EPT, SEL_THREADS / 32>(lg, t0, T, E, K, topk_idx, gates, logits_out, psum, sel_bias);
}

// out[i] = sum_{s < ks} part[s * n + i], in split order; four elements per
// thread when n allows, with the loads of four splits in flight at once.
__global__ void __launch_bounds__(128)
router_reduce_kernel(const float* __restrict__ part, int ks, size_t n, float* __restrict__ out) {
    pdl_wait();
    pdl_allow_next();
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    const size_t i0 = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if ((n & 3) == 0) {
        const size_t n4 = n >> 2;
        const float4* p4 = reinterpret_cast<const float4*>(part);
        for (size_t i = i0; i < n4; i += stride) {
            float4 s = __ldg(p4 + i);
            int k = 1;
            for (; k + 4 <= ks; k += 4) {
                float4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) v[u] = __ldg(p4 + static_cast<size_t>(k + u) * n4 + i);
#pragma unroll
                for (int u = 0; u < 4; ++u) { s.x += v[u].x; s.y += v[u].y; s.z += v[u].z; s.w += v[u].w; }
            }
            for (; k < ks; ++k) {
                const float4 v = __ldg(p4 + static_cast<size_t>(k) * n4 + i);
                s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
            }
            reinterpret_cast<float4*>(out)[i] = s;
        }
    } else {
        for (size_t i = i0; i < n; i += stride) {
            float s = part[i];
            for (int k = 1; k < ks; ++k) s += __ldg(part + static_cast<size_t>(k) * n + i);
            out[i] = s;
        }
    }
}

template <typename XT>
cudaError_t launch_generic(const Dims& dm, const void* x, const float* W_r, const float* bias,
                           int32_t* idx, float* gates, float* logits, float* psum, const float* sel_bias,
                           cudaStream_t st) {
    const dim3 grid(dm.route_blocks), block(NTHREADS);
    const XT* xp = static_cast<const XT*>(x);
    cudaError_t e;
#define MOE_GEN(EPT) e = launch_pdl(router_generic_kernel<XT, EPT>, grid, block, 0, st, 1, xp, W_r, bias, dm.T, dm.d, \
                                    dm.E, dm.K, idx, gates, logits, psum, sel_bias)
    if (dm.E <= 32) MOE_GEN(1);
    else if (dm.E <= 64) MOE_GEN(2);
    else if (dm.E <= 128) MOE_GEN(4);
    else MOE_GEN(8);
#undef MOE_GEN
    return e;
}

template <typename XT, int NE, int RT>
cudaError_t launch_small_t(const Dims& dm, const void* x, const float* W_r, const float* bias,
                           int32_t* idx, float* gates, float* logits, float* psum, int32_t* status,
                           const float* sel_bias, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(NE) * dm.d * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(router_small_kernel<XT, NE, RT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return launch_pdl(router_small_kernel<XT, NE, RT>, dim3(dm.route_blocks), dim3(SmallCfg<NE, RT>::WARPS * 32), smem,
                      st, 1, static_cast<const XT*>(x), W_r, bias, dm.T, dm.d, dm.E, dm.K, idx, gates, logits, psum,
                      status, sel_bias);
}

template <typename XT>
cudaError_t launch_small(const Dims& dm, const void* x, const float* W_r, const float* bias,
                         int32_t* idx, float* gates, float* logits, float* psum, int32_t* status,
                         const float* sel_bias, cudaStream_t st) {
    if (dm.E <= 8) return launch_small_t<XT, 8, 4>(dm, x, W_r, bias, idx, gates, logits, psum, status, sel_bias, st);
    if (dm.E <= 16) return launch_small_t<XT, 16, 4>(dm, x, W_r, bias, idx, gates, logits, psum, status, sel_bias, st);
    return launch_small_t<XT, 32, 2>(dm, x, W_r, bias, idx, gates, logits, psum, status, sel_bias, st);
}

}  // namespace

// The small kernel also serves long bf16 batches with few experts: the
// tensor-core router measured slower on the Mixtral shape (T = 4096, d =
// 4096, 8 experts: 25.6 against 22.5 us per call, same box), although the
// small kernel is latency-bound there (one 32-token block per SM, its FMA
// pipe a third busy, waiting on shared and global loads).
bool router_uses_small(const Dims& dm) {
    const int ne = dm.E <= 8 ? 8 : (dm.E <= 16 ? 16 : 32);
    return dm.E <= 32 && static_cast<size_t>(ne) * dm.d * 4 <= 160 * 1024;
}

bool router_uses_tc(const Dims& dm) {
    return !router_uses_small(dm) && dm.dtype != MOE_F32;
}

cudaError_t launch_router(const Dims& dm, const void* x, const float* W_r, const float* logit_bias,
                          int32_t* topk_idx, float* gates, float* logits_out, float* psum,
                          const RouterScratch& rs, cudaStream_t st) {
    // bias_mode 0: the bias enters the logits; 1: only the top-K keys
    const float* sel_bias = dm.bias_mode == 1 ? logit_bias : nullptr;
    if (dm.bias_mode == 1) logit_bias = nullptr;
    if (router_uses_small(dm)) {
        if (dm.dtype == MOE_F32)
            return launch_small<float>(dm, x, W_r, logit_bias, topk_idx, gates, logits_out, psum, rs.status,
                                       sel_bias, st);
        return launch_small<__nv_bfloat16>(dm, x, W_r, logit_bias, topk_idx, gates, logits_out, psum, rs.status,
                                           sel_bias, st);
    }
    if (!router_uses_tc(dm))
        return launch_generic<float>(dm, x, W_r, logit_bias, topk_idx, gates, logits_out, psum, sel_bias, st);
    const RouterTcPlan plan = router_tc_plan(dm);
    cudaError_t e = launch_router_tc(dm, plan, x, W_r, rs.w3, rs.part, rs.status, st);
    if (e != cudaSuccess) return e;
    // a few splits are summed by the select kernel as it loads them; many
    // are first reduced by a kernel spread over the whole GPU
    const float* logits = rs.part;
    int ks = plan.ksplit;
    if (ks > kSelectSplits) {
        const size_t n = static_cast<size_t>(dm.T) * dm.E;
        const size_t items = (n & 3) == 0 ? n / 4 : n;
        int blocks = static_cast<int>((items + 127) / 128);
        if (blocks > 8 * 148) blocks = 8 * 148;
        e = launch_pdl(router_reduce_kernel, dim3(blocks), dim3(128), 0, st, 1, static_cast<const float*>(rs.part), ks,
                       n, rs.logits);
        if (e != cudaSuccess) return e;
        logits = rs.logits;
        ks = 1;
    }
    const dim3 grid(dm.route_blocks), block(SEL_THREADS);
#define MOE_SEL(EPT) e = launch_pdl(router_select_kernel<EPT>, grid, block, 0, st, 1, logits, ks, logit_bias, dm.T, \
                                    dm.E, dm.K, topk_idx, gates, logits_out, psum, sel_bias)
    if (dm.E <= 32) MOE_SEL(1);
    else if (dm.E <= 64) MOE_SEL(2);
    else if (dm.E <= 128) MOE_SEL(4);
    else MOE_SEL(8);
#undef MOE_SEL
    return e;
}

}  // namespace moe

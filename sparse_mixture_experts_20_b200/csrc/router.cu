// Router: logits, softmax, top-K and gate renormalisation in one kernel.
//
// "論文解説: DeepSeekMoE" §ルーティングとバランス損失: s_j = softmax(W_r x)_j,
// g_j = s_j / sum_{k in TopK} s_k; §アルゴリズム: the router is a Linear
// layer without bias.  "Sparse MoE Top-Kルーティング" §ルーティングの仕組み.
//
// One block of 256 threads handles 32 tokens and every expert.  The logits
// are an fp32 GEMM (x tile x W_r^T) staged through shared memory in chunks of
// 32 columns; warp w then owns tokens w, w+8, w+16, w+24 and does the
// softmax, a K-round warp arg-max (ties to the lower expert index) and the
// gates with shuffles.  Per-block column sums of s go to psum in a fixed
// order, so the balance statistics are bit-reproducible.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int TT = kRouteTokens;   // tokens per block
constexpr int KC = 32;             // columns per shared-memory chunk
constexpr int NTHREADS = 256;

template <typename XT> __device__ __forceinline__ float to_f(XT v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename XT, int EPT>
__global__ void __launch_bounds__(NTHREADS)
router_kernel(const XT* __restrict__ x, const float* __restrict__ W_r,
              const float* __restrict__ logit_bias, int T, int d, int E, int K,
              int32_t* __restrict__ topk_idx, float* __restrict__ gates,
              float* __restrict__ logits_out, float* __restrict__ psum) {
    constexpr int NP = EPT * 32;                     // experts padded to the lanes
    __shared__ float xs[TT][KC + 1];
    __shared__ float wsh[(NP * (KC + 1) > TT * (NP + 1)) ? NP * (KC + 1) : TT * (NP + 1)];
    float (*wtile)[KC + 1] = reinterpret_cast<float (*)[KC + 1]>(wsh);
    float (*lg)[NP + 1] = reinterpret_cast<float (*)[NP + 1]>(wsh);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * TT;

    float acc[4][EPT];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < EPT; ++b) acc[a][b] = 0.f;

    for (int k0 = 0; k0 < d; k0 += KC) {
        // x chunk: TT x KC values, 4 per thread
#pragma unroll
        for (int i = 0; i < (TT * KC) / NTHREADS; ++i) {
            const int e = tid + i * NTHREADS;
            const int r = e / KC, c = e % KC;
            const int t = t0 + r;
            xs[r][c] = (t < T) ? to_f<XT>(x[static_cast<size_t>(t) * d + k0 + c]) : 0.f;
        }
        // W_r chunk: NP x KC values as float4
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

    // logits (+ bias) into shared memory; padded experts get -inf
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

    // per-token softmax / top-K / gates: warp w owns tokens w + 8*i
#pragma unroll 1
    for (int i = 0; i < TT / 8; ++i) {
        const int r = warp + 8 * i;
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
        uint32_t taken = 0;
        float vmax = 0.f, sel_v = 0.f;
        int sel_j = 0;
        for (int k = 0; k < K; ++k) {
            float bv = -INFINITY;
            int bj = 0x7fffffff;
#pragma unroll
            for (int b = 0; b < EPT; ++b) {
                const int j = lane + 32 * b;
                const bool ok = j < E && !((taken >> b) & 1u);
                if (ok && (v[b] > bv || (v[b] == bv && j < bj))) { bv = v[b]; bj = j; }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
                if (ov > bv || (ov == bv && oj < bj)) { bv = ov; bj = oj; }
            }
            if (k == 0) vmax = bv;
            if ((bj & 31) == lane) taken |= 1u << (bj >> 5);
            if (lane == k) { sel_v = bv; sel_j = bj; }
        }
        // softmax over all experts
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
        // gates: s_sel / sum s_sel over the K selected experts
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

    // per-block column sums of s, token order
    for (int j = tid; j < E; j += NTHREADS) {
        float s = 0.f;
        for (int r = 0; r < TT; ++r) s += lg[r][j];
        psum[static_cast<size_t>(blockIdx.x) * E + j] = s;
    }
}

template <typename XT>
cudaError_t launch_t(const Dims& dm, const void* x, const float* W_r, const float* bias,
                     int32_t* idx, float* gates, float* logits, float* psum, cudaStream_t st) {
    const dim3 grid(dm.route_blocks), block(NTHREADS);
    const XT* xp = static_cast<const XT*>(x);
    if (dm.E <= 32)
        router_kernel<XT, 1><<<grid, block, 0, st>>>(xp, W_r, bias, dm.T, dm.d, dm.E, dm.K, idx, gates, logits, psum);
    else if (dm.E <= 64)
        router_kernel<XT, 2><<<grid, block, 0, st>>>(xp, W_r, bias, dm.T, dm.d, dm.E, dm.K, idx, gates, logits, psum);
    else if (dm.E <= 128)
        router_kernel<XT, 4><<<grid, block, 0, st>>>(xp, W_r, bias, dm.T, dm.d, dm.E, dm.K, idx, gates, logits, psum);
    else
        router_kernel<XT, 8><<<grid, block, 0, st>>>(xp, W_r, bias, dm.T, dm.d, dm.E, dm.K, idx, gates, logits, psum);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const Dims& dm, const void* x, const float* W_r, const float* logit_bias,
                          int32_t* topk_idx, float* gates, float* logits_out, float* psum,
                          cudaStream_t st) {
    if (dm.dtype == MOE_F32)
        return launch_t<float>(dm, x, W_r, logit_bias, topk_idx, gates, logits_out, psum, st);
    return launch_t<__nv_bfloat16>(dm, x, W_r, logit_bias, topk_idx, gates, logits_out, psum, st);
}

}  // namespace moe

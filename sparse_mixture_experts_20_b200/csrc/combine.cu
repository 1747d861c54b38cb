// Combine and balance statistics.
//
// "論文解説: DeepSeekMoE" §共有エキスパート機構: h_t = sum_i E_s,i(x_t)
// + sum_{j in TopK} g_j E_r,j(x_t); §ルーティングとバランス損失:
// L = alpha * N_r * sum_j f_j P_j.  "DeepSeek DeepEP" §DeepEP とは item 5:
// BF16 combine.  "エキスパート並列（Expert Parallelism）" §推論フロー step 5:
// results return to their token (on one GPU: a gather).
//
// combine_kernel: warp(s) per token; each lane owns 16-byte chunks of the
// output row, gathers the token's kept expert rows (loads issued together,
// accumulated in ascending k) with 16-byte loads, accumulates g * y in fp32,
// adds the shared experts' rows (ascending s) and rounds once.
// balance_kernel: one block running balance_block (balance.cuh): chunked sums
// in a fixed order, so f, P and the loss are bit-reproducible.
#include "balance.cuh"
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {


constexpr int CB_WARPS = 8;       // warps per combine block
constexpr int kMaxWarpsPerToken = 32;

// W warps per token (W = 1 for large batches, up to 32 -- four blocks -- for
// small ones); global warp g serves token g / W, share g % W.  Lanes
// 0..K-1 read the token's slot rows and gates and broadcast them; each lane
// then owns 16-byte chunks of the output row: it issues the loads of all the
// token's kept rows for U chunks (U * KT = 8 rows' worth in flight when K is
// small) before accumulating each chunk in ascending k (then the shared rows
// in ascending s) in fp32, and rounds once.
template <bool F32, int KT, int U = (KT >= 8 ? 1 : 8 / KT)>   // KT >= K: register slots for the
__global__ void __launch_bounds__(32 * CB_WARPS, KT <= 8 ? 4 : 2)          // token's rows; U chunks per round
combine_kernel(const void* __restrict__ y_, const float* __restrict__ gates,
               const int32_t* __restrict__ slot_row, int T, int d, int K, int S, int r_cap,
               const void* __restrict__ x_, void* __restrict__ out_, int wpt) {
    pdl_wait();
    pdl_allow_next();
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * CB_WARPS + (threadIdx.x >> 5);
    const int t = gw / wpt;
    const int sub = gw % wpt;
    if (t >= T) return;
    const int my_row = lane < K ? slot_row[static_cast<size_t>(t) * K + lane] : -1;
    const float my_g = lane < K ? gates[static_cast<size_t>(t) * K + lane] : 0.f;
    int rows[KT];
    float g[KT];
#pragma unroll
    for (int k = 0; k < KT; ++k) {
        rows[k] = __shfl_sync(0xffffffffu, my_row, k);
        g[k] = __shfl_sync(0xffffffffu, my_g, k);
    }
    const int nchunks = d / (F32 ? 4 : 8);
    const uint4* y = static_cast<const uint4*>(y_);          // rows of nchunks 16-byte chunks
    uint4* out = static_cast<uint4*>(out_) + static_cast<size_t>(t) * nchunks;
    // a kept slot reads its expert row; with pass-through (x_ != nullptr) a
    // slot dropped by the capacity (row -1) reads the token's own input
    const uint4* xr = static_cast<const uint4*>(x_);
    const int stride = 32 * wpt;                             // chunks between a lane's consecutive chunks
    for (int c0 = sub * 32 + lane; c0 < nchunks; c0 += U * stride) {
        // the loads of U chunks of all K rows are issued before any is used
        uint4 raw[U][KT];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * stride;
            const bool in = c < nchunks;
#pragma unroll
            for (int k = 0; k < KT; ++k)
                raw[u][k] = (in && k < K && rows[k] >= 0) ? __ldg(y + static_cast<size_t>(rows[k]) * nchunks + c)
                            : (in && k < K && rows[k] == -1 && xr != nullptr)
                                ? __ldg(xr + static_cast<size_t>(t) * nchunks + c)
                                : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * stride;
            if (c >= nchunks) break;
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
            for (int k = 0; k < KT; ++k) {
                if (k >= K || rows[k] < -1 || (rows[k] == -1 && xr == nullptr)) continue;
                if (F32) {
                    const float* f = reinterpret_cast<const float*>(&raw[u][k]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[i] = fmaf(g[k], f[i], acc[i]);
                } else {
                    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u][k]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 f = __bfloat1622float2(h2[i]);
                        acc[2 * i] = fmaf(g[k], f.x, acc[2 * i]);
                        acc[2 * i + 1] = fmaf(g[k], f.y, acc[2 * i + 1]);
                    }
                }
            }
            for (int s = 0; s < S; ++s) {
                const uint4 v = __ldg(y + (static_cast<size_t>(r_cap) + static_cast<size_t>(s) * T + t) * nchunks + c);
                if (F32) {
                    const float* f = reinterpret_cast<const float*>(&v);
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[i] += f[i];
                } else {
                    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 f = __bfloat1622float2(h2[i]);
                        acc[2 * i] += f.x;
                        acc[2 * i + 1] += f.y;
                    }
                }
            }
            uint4 o;
            if (F32) {
                o = make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                               __float_as_uint(acc[3]));
            } else {
                uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
                    ow[i] = *reinterpret_cast<uint32_t*>(&v);
                }
            }
            out[c] = o;
        }
    }
}

__global__ void __launch_bounds__(BALANCE_THREADS)
balance_kernel(const int32_t* __restrict__ counts, const float* __restrict__ psum, int blocks,
               int T, int E, int K, float alpha, float* __restrict__ f, float* __restrict__ P,
               float* __restrict__ loss) {
    __shared__ float part[BALANCE_THREADS];
    __shared__ float fp[256];
    pdl_wait();
    pdl_allow_next();
    balance_block(counts, psum, blocks, T, E, K, alpha, f, P, loss, part, fp);
}

}  // namespace

cudaError_t launch_combine(const Dims& dm, const void* y, const float* gates,
                           const int32_t* slot_row, const void* x, void* out, cudaStream_t st) {
    if (!dm.passthrough) x = nullptr;
    const bool f32 = dm.dtype == MOE_F32;
    int wpt = 1;                              // enough warps in flight to fill the GPU at small T
    while (wpt < kMaxWarpsPerToken && static_cast<long long>(dm.T) * wpt < 148LL * 32) wpt *= 2;
    const int blocks = static_cast<int>((static_cast<long long>(dm.T) * wpt + CB_WARPS - 1) / CB_WARPS);
    cudaError_t e;
#define MOE_COMBINE(F, KT) e = launch_pdl(combine_kernel<F, KT>, dim3(blocks), dim3(32 * CB_WARPS), 0, st, 1, \
        y, gates, slot_row, dm.T, dm.d, dm.K, dm.S, dm.r_cap, x, out, wpt)
#define MOE_COMBINE_K(F)                                                                         \
    if (dm.K <= 2) MOE_COMBINE(F, 2);                                                            \
    else if (dm.K <= 4) MOE_COMBINE(F, 4);                                                       \
    else if (dm.K <= 8) MOE_COMBINE(F, 8);                                                       \
    else MOE_COMBINE(F, 16)
    if (f32) { MOE_COMBINE_K(true); }
    else { MOE_COMBINE_K(false); }
#undef MOE_COMBINE_K
#undef MOE_COMBINE
    return e;
}

cudaError_t launch_balance(const Dims& dm, const int32_t* counts, const float* psum,
                           float* f, float* P, float* loss, cudaStream_t st) {
    return launch_pdl(balance_kernel, dim3(1), dim3(BALANCE_THREADS), 0, st, 1, counts, psum, dm.route_blocks, dm.T, dm.E,
                      dm.K, dm.alpha, f, P, loss);
}

}  // namespace moe

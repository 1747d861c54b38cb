// Combine and balance statistics.
//
// "論文解説: DeepSeekMoE" §共有エキスパート機構: h_t = sum_i E_s,i(x_t)
// + sum_{j in TopK} g_j E_r,j(x_t); §ルーティングとバランス損失:
// L = alpha * N_r * sum_j f_j P_j.  "DeepSeek DeepEP" §DeepEP とは item 5:
// BF16 combine.  "エキスパート並列（Expert Parallelism）" §推論フロー step 5:
// results return to their token (on one GPU: a gather).
//
// combine_kernel: block per token; each thread owns 16 bytes of the output
// row, gathers the token's kept expert rows (ascending k) with 16-byte loads,
// accumulates g * y in fp32, adds the shared experts' rows (ascending s) and
// rounds once.
// balance_kernel: one block; fixed-order reductions, so f, P and the loss are
// bit-reproducible.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int MAXK = 16;

template <bool F32>
__global__ void __launch_bounds__(1024)
combine_kernel(const void* __restrict__ y_, const float* __restrict__ gates,
               const int32_t* __restrict__ slot_row, int T, int d, int K, int S, int r_cap,
               void* __restrict__ out_) {
    __shared__ int rows_s[MAXK];
    __shared__ float g_s[MAXK];
    const int t = blockIdx.x, tid = threadIdx.x;
    if (tid < K) {
        rows_s[tid] = slot_row[static_cast<size_t>(t) * K + tid];
        g_s[tid] = gates[static_cast<size_t>(t) * K + tid];
    }
    __syncthreads();
    if (F32) {
        const float* y = static_cast<const float*>(y_);
        for (int c = tid; c < d / 4; c += blockDim.x) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int k = 0; k < K; ++k) {
                const int r = rows_s[k];
                if (r < 0) continue;
                const float g = g_s[k];
                const float4 v = reinterpret_cast<const float4*>(y + static_cast<size_t>(r) * d)[c];
                acc.x = fmaf(g, v.x, acc.x); acc.y = fmaf(g, v.y, acc.y);
                acc.z = fmaf(g, v.z, acc.z); acc.w = fmaf(g, v.w, acc.w);
            }
            for (int s = 0; s < S; ++s) {
                const float4 v = reinterpret_cast<const float4*>(
                    y + (static_cast<size_t>(r_cap) + static_cast<size_t>(s) * T + t) * d)[c];
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
            reinterpret_cast<float4*>(static_cast<float*>(out_) + static_cast<size_t>(t) * d)[c] = acc;
        }
    } else {
        const __nv_bfloat16* y = static_cast<const __nv_bfloat16*>(y_);
        for (int c = tid; c < d / 8; c += blockDim.x) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            for (int k = 0; k < K; ++k) {
                const int r = rows_s[k];
                if (r < 0) continue;
                const float g = g_s[k];
                const uint4 raw = __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(r) * d) + c);
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(h2[i]);
                    acc[2 * i] = fmaf(g, f.x, acc[2 * i]);
                    acc[2 * i + 1] = fmaf(g, f.y, acc[2 * i + 1]);
                }
            }
            for (int s = 0; s < S; ++s) {
                const uint4 raw = __ldg(reinterpret_cast<const uint4*>(
                    y + (static_cast<size_t>(r_cap) + static_cast<size_t>(s) * T + t) * d) + c);
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(h2[i]);
                    acc[2 * i] += f.x;
                    acc[2 * i + 1] += f.y;
                }
            }
            uint4 o;
            uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
                ow[i] = *reinterpret_cast<uint32_t*>(&v);
            }
            reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out_) + static_cast<size_t>(t) * d)[c] = o;
        }
    }
}

__global__ void __launch_bounds__(256)
balance_kernel(const int32_t* __restrict__ counts, const float* __restrict__ psum, int blocks,
               int T, int E, int K, float alpha, float* __restrict__ f, float* __restrict__ P,
               float* __restrict__ loss) {
    __shared__ float fp[256];
    const int j = threadIdx.x;
    float prod = 0.f;
    if (j < E) {
        float s = 0.f;
        for (int b = 0; b < blocks; ++b) s += psum[static_cast<size_t>(b) * E + j];
        const float fj = static_cast<float>(counts[j]) / static_cast<float>(T * K);
        const float pj = s / static_cast<float>(T);
        f[j] = fj;
        P[j] = pj;
        prod = fj * pj;
    }
    fp[j] = prod;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (j < w) fp[j] += fp[j + w];
        __syncthreads();
    }
    if (j == 0) *loss = alpha * static_cast<float>(E) * fp[0];
}

}  // namespace

cudaError_t launch_combine(const Dims& dm, const void* y, const float* gates,
                           const int32_t* slot_row, void* out, cudaStream_t st) {
    const bool f32 = dm.dtype == MOE_F32;
    int threads = dm.d / (f32 ? 4 : 8);
    if (threads > 1024) threads = 1024;
    threads = (threads + 31) / 32 * 32;
    if (f32) combine_kernel<true><<<dm.T, threads, 0, st>>>(y, gates, slot_row, dm.T, dm.d, dm.K, dm.S, dm.r_cap, out);
    else combine_kernel<false><<<dm.T, threads, 0, st>>>(y, gates, slot_row, dm.T, dm.d, dm.K, dm.S, dm.r_cap, out);
    count_launches();
    return cudaGetLastError();
}

cudaError_t launch_balance(const Dims& dm, const int32_t* counts, const float* psum,
                           float* f, float* P, float* loss, cudaStream_t st) {
    balance_kernel<<<1, 256, 0, st>>>(counts, psum, dm.route_blocks, dm.T, dm.E, dm.K, dm.alpha, f, P, loss);
    count_launches();
    return cudaGetLastError();
}

}  // namespace moe

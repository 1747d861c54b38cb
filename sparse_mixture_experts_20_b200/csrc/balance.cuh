// Balance statistics of one batch, computed by one block of BALANCE_THREADS
// threads ("論文解説: DeepSeekMoE" §ルーティングとバランス損失:
// f_j = counts_j / (T K), P_j = mean over tokens of s_j, L = alpha N_r sum f_j P_j).
//
// Thread (c, j) = (tid / E, tid % E) sums the per-router-block partial sums
// of s of expert j over its chunk c of the router blocks, eight loads in
// flight at a time; the C chunk sums of each expert are then added in chunk
// order and the products f_j P_j in a fixed tree, so f, P and the loss are
// bit-reproducible -- and the same wherever this routine runs (the balance
// kernel, or the end of the dispatch scan inside moe_layer_forward).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int BALANCE_THREADS = 1024;

// part: BALANCE_THREADS floats, fp: 256 floats of shared memory.  counts may
// have been written by this block (visible after the block barrier inside).
__device__ __forceinline__ void balance_block(const int32_t* counts, const float* __restrict__ psum, int blocks,
                                              int T, int E, int K, float alpha, float* __restrict__ f,
                                              float* __restrict__ P, float* __restrict__ loss, float* part,
                                              float* fp) {
    const int tid = threadIdx.x;
    const int C = BALANCE_THREADS / E;                   // >= 4: E <= 256
    const int c = tid / E, j = tid - c * E;
    if (c < C) {
        const int b0 = static_cast<int>(static_cast<long long>(c) * blocks / C);
        const int b1 = static_cast<int>(static_cast<long long>(c + 1) * blocks / C);
        float s = 0.f;
        int b = b0;
        for (; b + 8 <= b1; b += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldg(psum + static_cast<size_t>(b + u) * E + j);
#pragma unroll
            for (int u = 0; u < 8; ++u) s += v[u];
        }
        for (; b < b1; ++b) s += __ldg(psum + static_cast<size_t>(b) * E + j);
        part[tid] = s;
    }
    __syncthreads();
    if (tid < 256) {
        float prod = 0.f;
        if (tid < E) {
            float s = 0.f;
            for (int q = 0; q < C; ++q) s += part[q * E + tid];
            const float fj = static_cast<float>(counts[tid]) / static_cast<float>(T * K);
            const float pj = s / static_cast<float>(T);
            f[tid] = fj;
            P[tid] = pj;
            prod = fj * pj;
        }
        fp[tid] = prod;
    }
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (tid < w) fp[tid] += fp[tid + w];
        __syncthreads();
    }
    if (tid == 0) *loss = alpha * static_cast<float>(E) * fp[0];
}

}  // namespace moe

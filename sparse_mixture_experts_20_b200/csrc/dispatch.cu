// Dispatch: the single-GPU form of the expert-parallel token exchange.
//
// "エキスパート並列（Expert Parallelism）" §推論フロー: after the gate picks the
// experts, tokens travel to the expert that serves them.  On one GPU that
// all-to-all is a permutation of rows into per-expert segments.
// "Sparse MoE Top-Kルーティング" §解決策2 and FAQ Q2: an expert takes at most
// C tokens per batch; the rest are dropped.  "DeepSeek DeepEP" §DeepEP とは
// item 5: tokens are dispatched in FP8.
//
// Three kernels, no atomics, deterministic:
//   1. bitmap_kernel : warp per 32 tokens; for each expert j a ballot gives
//      the 32-bit mask of those tokens that selected j -> bitmap[word][j].
//      Out-of-range or repeated indices set MOE_DEV_BAD_ROUTING and are
//      ignored.
//   2. scan_kernel   : one block; per expert, prefix sums of popcounts over
//      words -> word_base[word][j] (slots of j in earlier words), counts,
//      kept = min(counts, C), offsets = exclusive scan of kept.
//   3. scatter_kernel: block per token; thread k < K finds the slot's rank
//      (word_base + popcount of the lower lanes' bits), keeps it if rank < C,
//      writes slot_row / row_slot; then the block copies (bf16/fp32) or
//      quantises to e4m3 (FP8) the token's row into each kept destination
//      with 16-byte accesses.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// A slot is valid if its expert index is in range and not repeated by an
// earlier slot of the same token.  `ids` holds the token's K indices.
__device__ __forceinline__ bool slot_valid(const int* ids, int k, int E) {
    const int j = ids[k];
    if (j < 0 || j >= E) return false;
    for (int q = 0; q < k; ++q)
        if (ids[q] == j) return false;
    return true;
}

constexpr int MAXK = 16;

__global__ void __launch_bounds__(256)
bitmap_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int K, int t_words,
              uint32_t* __restrict__ bitmap, int32_t* status) {
    const int lane = threadIdx.x & 31;
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (w >= t_words) return;
    const int t = w * 32 + lane;
    int ids[MAXK];
    bool bad = false;
#pragma unroll
    for (int k = 0; k < MAXK; ++k) {
        ids[k] = -1;
        if (k < K && t < T) ids[k] = topk_idx[static_cast<size_t>(t) * K + k];
    }
    int valid[MAXK];
#pragma unroll
    for (int k = 0; k < MAXK; ++k) {
        valid[k] = -1;
        if (k < K && t < T) {
            if (slot_valid(ids, k, E)) valid[k] = ids[k];
            else bad = true;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_device_status(status, MOE_DEV_BAD_ROUTING);
    for (int j0 = 0; j0 < E; j0 += 32) {
        uint32_t mine = 0;
        for (int jj = 0; jj < 32 && j0 + jj < E; ++jj) {
            const int j = j0 + jj;
            bool hit = false;
#pragma unroll
            for (int k = 0; k < MAXK; ++k) hit |= (valid[k] == j);
            const uint32_t m = __ballot_sync(0xffffffffu, hit);
            if (lane == jj) mine = m;
        }
        if (j0 + lane < E) bitmap[static_cast<size_t>(w) * E + j0 + lane] = mine;
    }
}

// One block of 1024 threads.  Thread (j, p): expert j, word slice p of P.
__global__ void __launch_bounds__(1024)
scan_kernel(const uint32_t* __restrict__ bitmap, int E, int t_words, int capacity,
            int32_t* __restrict__ word_base, int32_t* __restrict__ counts,
            int32_t* __restrict__ kept, int32_t* __restrict__ offsets) {
    __shared__ int part[1024];
    __shared__ int kept_s[256];
    int P = 1;
    while (P * 2 * E <= 1024 && P < 128) P *= 2;
    const int tid = threadIdx.x;
    const int j = tid / P, p = tid % P;
    const int wpp = (t_words + P - 1) / P;
    const int w0 = p * wpp, w1 = min(t_words, w0 + wpp);
    int sum = 0;
    if (j < E)
        for (int w = w0; w < w1; ++w) sum += __popc(bitmap[static_cast<size_t>(w) * E + j]);
    part[tid] = sum;
    __syncthreads();
    if (j < E && p == 0) {                  // exclusive scan over the P slices of expert j
        int run = 0;
        for (int q = 0; q < P; ++q) {
            const int v = part[tid + q];
            part[tid + q] = run;
            run += v;
        }
        counts[j] = run;
        kept_s[j] = (capacity >= 0) ? min(run, capacity) : run;
    }
    __syncthreads();
    if (j < E) {
        int run = part[tid];
        for (int w = w0; w < w1; ++w) {
            word_base[static_cast<size_t>(w) * E + j] = run;
            run += __popc(bitmap[static_cast<size_t>(w) * E + j]);
        }
    }
    if (tid < 32) {                         // offsets = exclusive scan of kept (warp 0)
        int carry = 0;
        for (int base = 0; base < E; base += 32) {
            const int i = base + tid;
            int v = (i < E) ? kept_s[i] : 0;
            if (i < E) kept[i] = v;
            int incl = v;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (tid >= off) incl += o;
            }
            if (i < E) offsets[i] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (tid == 0) offsets[E] = carry;
    }
}

template <int MODE>   // 0: fp32 copy, 1: bf16 copy, 2: bf16 -> e4m3 + 1x128 scales
__global__ void __launch_bounds__(1024)
scatter_kernel(const void* __restrict__ x_, const int32_t* __restrict__ topk_idx,
               const uint32_t* __restrict__ bitmap, const int32_t* __restrict__ word_base,
               const int32_t* __restrict__ offsets, int T, int d, int E, int K, int capacity,
               int r_cap, int shared_copy, int32_t* __restrict__ slot_row,
               int32_t* __restrict__ row_slot, void* __restrict__ x_disp_,
               float* __restrict__ x_disp_scales) {
    __shared__ int rows_s[MAXK];
    const int t = blockIdx.x;
    const int tid = threadIdx.x;
    if (tid < K) {
        int ids[MAXK];
        for (int k = 0; k < K; ++k) ids[k] = topk_idx[static_cast<size_t>(t) * K + k];
        int row = -1;
        if (slot_valid(ids, tid, E)) {
            const int j = ids[tid];
            const int w = t >> 5;
            const uint32_t below = bitmap[static_cast<size_t>(w) * E + j] & ((1u << (t & 31)) - 1u);
            const int rank = word_base[static_cast<size_t>(w) * E + j] + __popc(below);
            if (capacity < 0 || rank < capacity) row = offsets[j] + rank;
        }
        rows_s[tid] = row;
        slot_row[static_cast<size_t>(t) * K + tid] = row;
        if (row >= 0) row_slot[row] = t * K + tid;
    }
    __syncthreads();
    if (MODE == 0) {
        const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x_) + static_cast<size_t>(t) * d);
        for (int c = tid; c < d / 4; c += blockDim.x) {
            const float4 v = src[c];
            for (int k = 0; k < K; ++k) {
                const int r = rows_s[k];
                if (r >= 0) reinterpret_cast<float4*>(static_cast<float*>(x_disp_) + static_cast<size_t>(r) * d)[c] = v;
            }
        }
    } else if (MODE == 1) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x_) + static_cast<size_t>(t) * d);
        for (int c = tid; c < d / 8; c += blockDim.x) {
            const uint4 v = src[c];
            for (int k = 0; k < K; ++k) {
                const int r = rows_s[k];
                if (r >= 0) reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(x_disp_) + static_cast<size_t>(r) * d)[c] = v;
            }
        }
    } else {
        // 16 consecutive threads own one 128-column block (8 values each);
        // blockDim is a multiple of 16 and d a multiple of 128.
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x_) + static_cast<size_t>(t) * d);
        uint8_t* xd = static_cast<uint8_t*>(x_disp_);
        const int nq = d / 128;
        const int nchunks = d / 8;
        // every lane runs every round so that the 16-lane shuffles are full-warp
        for (int base = 0; base < nchunks; base += blockDim.x) {
            const int c = base + tid;
            const bool act = c < nchunks;
            float v[8];
            if (act) {
                const uint4 raw = src[c];
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(h2[i]);
                    v[2 * i] = f.x;
                    v[2 * i + 1] = f.y;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = 0.f;
            }
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off, 16));
            if (!act) continue;
            const float sc = pow2_scale_448(amax);
            const float inv = 1.0f / sc;                     // exact: power of two
            uint2 q;
            q.x = static_cast<uint32_t>(f32x2_to_e4m3x2(v[0] * inv, v[1] * inv)) |
                  (static_cast<uint32_t>(f32x2_to_e4m3x2(v[2] * inv, v[3] * inv)) << 16);
            q.y = static_cast<uint32_t>(f32x2_to_e4m3x2(v[4] * inv, v[5] * inv)) |
                  (static_cast<uint32_t>(f32x2_to_e4m3x2(v[6] * inv, v[7] * inv)) << 16);
            const int blk = c >> 4;
            const bool lead = (c & 15) == 0;
            for (int k = 0; k <= K; ++k) {
                int r;
                if (k < K) r = rows_s[k];
                else r = shared_copy ? r_cap + t : -1;
                if (r < 0) continue;
                reinterpret_cast<uint2*>(xd + static_cast<size_t>(r) * d)[c] = q;
                if (lead) x_disp_scales[static_cast<size_t>(r) * nq + blk] = sc;
            }
        }
    }
}

}  // namespace

cudaError_t launch_dispatch(const Dims& dm, const void* x, const int32_t* topk_idx,
                            int32_t* counts, int32_t* kept, int32_t* offsets,
                            int32_t* slot_row, int32_t* row_slot, void* x_disp,
                            float* x_disp_scales, uint32_t* bitmap, int32_t* word_base,
                            int32_t* status, cudaStream_t st) {
    bitmap_kernel<<<(dm.t_words + 7) / 8, 256, 0, st>>>(topk_idx, dm.T, dm.E, dm.K, dm.t_words, bitmap, status);
    scan_kernel<<<1, 1024, 0, st>>>(bitmap, dm.E, dm.t_words, dm.capacity, word_base, counts, kept, offsets);
    const int vec = dm.dtype == MOE_F32 ? 4 : 8;
    int threads = dm.d / vec;
    if (threads > 1024) threads = 1024;
    if (dm.dtype == MOE_FP8_E4M3_BLOCK) threads = threads / 16 * 16;
    threads = (threads + 31) / 32 * 32;
    const int shared_copy = (dm.dtype == MOE_FP8_E4M3_BLOCK && dm.S > 0) ? 1 : 0;
#define MOE_SCATTER(MODE) scatter_kernel<MODE><<<dm.T, threads, 0, st>>>(                 \
        x, topk_idx, bitmap, word_base, offsets, dm.T, dm.d, dm.E, dm.K, dm.capacity,      \
        dm.r_cap, shared_copy, slot_row, row_slot, x_disp, x_disp_scales)
    if (dm.dtype == MOE_F32) MOE_SCATTER(0);
    else if (dm.dtype == MOE_BF16) MOE_SCATTER(1);
    else MOE_SCATTER(2);
#undef MOE_SCATTER
    count_launches(3);
    return cudaGetLastError();
}

}  // namespace moe

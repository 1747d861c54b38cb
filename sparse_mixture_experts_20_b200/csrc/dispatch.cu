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
//   3. scatter_kernel: warp per token; lane k < K finds the slot's rank
//      (word_base + popcount of the lower lanes' bits), keeps it if rank < C,
//      writes slot_row / row_slot; then the warp copies (bf16/fp32) or
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
bitmap_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int K, int t_words, int planes,
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
    // planes == 1: one bitmap per word (any slot); planes == K: one per slot
    // index (slot-major capacity priority), plane p holding the p-th choices
    for (int pl = 0; pl < planes; ++pl) {
        for (int j0 = 0; j0 < E; j0 += 32) {
            uint32_t mine = 0;
            for (int jj = 0; jj < 32 && j0 + jj < E; ++jj) {
                const int j = j0 + jj;
                bool hit = false;
                if (planes == 1) {
#pragma unroll
                    for (int k = 0; k < MAXK; ++k) hit |= (valid[k] == j);
                } else {
#pragma unroll
                    for (int k = 0; k < MAXK; ++k) hit |= (k == pl && valid[k] == j);
                }
                const uint32_t m = __ballot_sync(0xffffffffu, hit);
                if (lane == jj) mine = m;
            }
            if (j0 + lane < E) bitmap[(static_cast<size_t>(pl) * t_words + w) * E + j0 + lane] = mine;
        }
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

constexpr int SC_WARPS = 8;       // warps per scatter block

// W warps per token (W = 1 for large batches; up to 8 when there are too few
// tokens to fill the GPU).  Lanes 0..K-1 resolve the token's K slots to destination
// rows (rank = word_base + popcount of the earlier tokens' bits of the word);
// the rows are broadcast with shuffles and the warp copies (bf16 / fp32) or
// quantises to e4m3 (FP8) the token's row into every kept destination with
// 16-byte (8-byte for e4m3) accesses.  The first loads of the row are issued
// before the slot resolution, so the two latencies overlap.
template <int MODE>   // 0: fp32 copy, 1: bf16 copy, 2: bf16 -> e4m3 + 1x128 scales
__global__ void __launch_bounds__(32 * SC_WARPS)
scatter_kernel(const void* __restrict__ x_, const int32_t* __restrict__ topk_idx,
               const uint32_t* __restrict__ bitmap, const int32_t* __restrict__ word_base,
               const int32_t* __restrict__ offsets, int T, int d, int E, int K, int capacity,
               int r_cap, int shared_copy, int32_t* __restrict__ slot_row,
               int32_t* __restrict__ row_slot, void* __restrict__ x_disp_,
               float* __restrict__ x_disp_scales, int wpt, int t_words, int slot_major) {
    constexpr int PF = 4;                                  // 16-byte chunks per lane in flight
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int t = blockIdx.x * (SC_WARPS / wpt) + warp / wpt;
    const int sub = warp % wpt;                            // this warp's share of the row
    if (t >= T) return;
    const int lane0 = sub * 32 + lane;                     // chunk of the first round
    const int stride = 32 * wpt;                           // chunks between rounds
    const int nchunks = d / (MODE == 0 ? 4 : 8);           // 16-byte chunks of the source row
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(x_) +
                                                      static_cast<size_t>(t) * d * (MODE == 0 ? 4 : 2));
    uint4 pre[PF];
#pragma unroll
    for (int u = 0; u < PF; ++u) {
        const int c = lane0 + stride * u;
        pre[u] = c < nchunks ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }
    // ---- slot resolution (lane k: slot k)
    const int my_id = lane < K ? topk_idx[static_cast<size_t>(t) * K + lane] : -1;
    int row = -2;                                          // -2: invalid index, -1: over the capacity
    {
        bool valid = lane < K && my_id >= 0 && my_id < E;
        for (int q = 0; q < K; ++q) {                      // repeated by an earlier slot?
            const int other = __shfl_sync(0xffffffffu, my_id, q);
            if (q < lane && other == my_id) valid = false;
        }
        if (valid) {
            // bitmap word: (plane, word); plane = the slot index under slot-major priority
            const size_t qw = static_cast<size_t>(slot_major ? lane : 0) * t_words + (t >> 5);
            const uint32_t below = bitmap[qw * E + my_id] & ((1u << (t & 31)) - 1u);
            const int rank = word_base[qw * E + my_id] + __popc(below);
            row = (capacity < 0 || rank < capacity) ? offsets[my_id] + rank : -1;
        }
        if (lane < K && sub == 0) {
            slot_row[static_cast<size_t>(t) * K + lane] = row;
            if (row >= 0) row_slot[row] = t * K + lane;
        }
    }
    int rows[MAXK + 1];
#pragma unroll
    for (int k = 0; k < MAXK; ++k) rows[k] = __shfl_sync(0xffffffffu, row, k);
    rows[MAXK] = (MODE == 2 && shared_copy) ? r_cap + t : -1;
    if (MODE != 2) {
        uint4* dst0 = static_cast<uint4*>(x_disp_);
        const size_t row_chunks = static_cast<size_t>(nchunks);
        for (int base = 0; base < nchunks; base += stride * PF) {
            uint4 v[PF];
#pragma unroll
            for (int u = 0; u < PF; ++u) {
                const int c = base + lane0 + stride * u;
                v[u] = base == 0 ? pre[u] : (c < nchunks ? __ldg(src + c) : make_uint4(0, 0, 0, 0));
            }
#pragma unroll
            for (int k = 0; k < MAXK; ++k) {
                if (k >= K) break;
                const int r = rows[k];
                if (r < 0) continue;
#pragma unroll
                for (int u = 0; u < PF; ++u) {
                    const int c = base + lane0 + stride * u;
                    if (c < nchunks) dst0[static_cast<size_t>(r) * row_chunks + c] = v[u];
                }
            }
        }
    } else {
        // 16 consecutive lanes own one 128-column block (8 values each); d is
        // a multiple of 128, so a 16-lane group is always entirely in range
        uint8_t* xd = static_cast<uint8_t*>(x_disp_);
        const int nq = d / 128;
        for (int base = 0; base < nchunks; base += stride * PF) {
            uint4 raw[PF];
#pragma unroll
            for (int u = 0; u < PF; ++u) {
                const int c = base + lane0 + stride * u;
                raw[u] = base == 0 ? pre[u] : (c < nchunks ? __ldg(src + c) : make_uint4(0, 0, 0, 0));
            }
#pragma unroll
            for (int u = 0; u < PF; ++u) {
                const int c = base + lane0 + stride * u;
                float v[8];
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
                for (int i2 = 0; i2 < 4; ++i2) {
                    const float2 f = __bfloat1622float2(h2[i2]);
                    v[2 * i2] = f.x;
                    v[2 * i2 + 1] = f.y;
                }
                float amax = 0.f;
#pragma unroll
                for (int i2 = 0; i2 < 8; ++i2) amax = fmaxf(amax, fabsf(v[i2]));
#pragma unroll
                for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off, 16));
                if (c >= nchunks) continue;
                const float sc = pow2_scale_448(amax);
                const float inv = inv_pow2(sc);                  // exact: power of two
                uint2 q;
                q.x = static_cast<uint32_t>(f32x2_to_e4m3x2(v[0] * inv, v[1] * inv)) |
                      (static_cast<uint32_t>(f32x2_to_e4m3x2(v[2] * inv, v[3] * inv)) << 16);
                q.y = static_cast<uint32_t>(f32x2_to_e4m3x2(v[4] * inv, v[5] * inv)) |
                      (static_cast<uint32_t>(f32x2_to_e4m3x2(v[6] * inv, v[7] * inv)) << 16);
                const int blk = c >> 4;
                const bool lead = (c & 15) == 0;
#pragma unroll
                for (int k = 0; k <= MAXK; ++k) {
                    if (k < MAXK && k >= K) continue;
                    const int r = rows[k];
                    if (r < 0) continue;
                    reinterpret_cast<uint2*>(xd + static_cast<size_t>(r) * d)[c] = q;
                    if (lead) x_disp_scales[static_cast<size_t>(r) * nq + blk] = sc;
                }
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
    bitmap_kernel<<<(dm.t_words + 7) / 8, 256, 0, st>>>(topk_idx, dm.T, dm.E, dm.K, dm.t_words, dm.planes,
                                                        bitmap, status);
    // the scan runs over the (plane, word) sequence: token order within a
    // plane, planes in slot order
    scan_kernel<<<1, 1024, 0, st>>>(bitmap, dm.E, dm.planes * dm.t_words, dm.capacity, word_base, counts, kept,
                                    offsets);
    const int shared_copy = (dm.dtype == MOE_FP8_E4M3_BLOCK && dm.S > 0) ? 1 : 0;
    // warps per token: enough warps in flight to fill the GPU at small T
    int wpt = 1;
    while (wpt < SC_WARPS && static_cast<long long>(dm.T) * wpt < 148LL * 32) wpt *= 2;
    const int tpb = SC_WARPS / wpt;
    const int blocks = (dm.T + tpb - 1) / tpb;
#define MOE_SCATTER(MODE) scatter_kernel<MODE><<<blocks, 32 * SC_WARPS, 0, st>>>(          \
        x, topk_idx, bitmap, word_base, offsets, dm.T, dm.d, dm.E, dm.K, dm.capacity,      \
        dm.r_cap, shared_copy, slot_row, row_slot, x_disp, x_disp_scales, wpt, dm.t_words, dm.slot_major)
    if (dm.dtype == MOE_F32) MOE_SCATTER(0);
    else if (dm.dtype == MOE_BF16) MOE_SCATTER(1);
    else MOE_SCATTER(2);
#undef MOE_SCATTER
    count_launches(3);
    return cudaGetLastError();
}

}  // namespace moe

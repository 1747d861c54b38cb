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
//   1. bitmap_kernel : warp per 32 tokens; lane i ORs bit i into the mask of
//      each expert its token selected (shared memory), giving the 32-bit mask
//      of the word's tokens that selected j -> bitmap[word][j].
//      Out-of-range or repeated indices set MOE_DEV_BAD_ROUTING and are
//      ignored.
//   2. scan_kernel   : one block; per expert, prefix sums of popcounts over
//      words -> word_base[word][j] (slots of j in earlier words), counts,
//      kept = min(counts, C), offsets = exclusive scan of kept (parallel
//      scans over word slices and over experts).
//   3. scatter_kernel: warp(s) per token; lane k < K finds the slot's rank
//      (word_base + popcount of the lower lanes' bits), keeps it if rank < C,
//      writes slot_row / row_slot; then the warp copies (bf16/fp32) or
//      quantises to e4m3 (FP8) the token's row into each kept destination
//      with 16-byte accesses.
#include "balance.cuh"
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

// Warp per 32-token word.  The word's masks (planes * E of them) are built in
// this warp's slice of shared memory by atomicOr -- K operations per lane
// instead of a ballot per expert; OR does not depend on the order, so the
// result is deterministic -- and then written out coalesced.
__global__ void __launch_bounds__(256)
bitmap_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int K, int t_words, int planes,
              uint32_t* __restrict__ bitmap, int32_t* status) {
    extern __shared__ uint32_t bm_s[];                    // (warps of the block, planes * E)
    pdl_wait();
    pdl_allow_next();
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int w = blockIdx.x * (blockDim.x >> 5) + wib;
    if (w >= t_words) return;                             // whole warps only; no block barrier below
    const int words = planes * E;
    uint32_t* sm = bm_s + static_cast<size_t>(wib) * words;
    for (int i = lane; i < words; i += 32) sm[i] = 0u;
    const int t = w * 32 + lane;
    int ids[MAXK];
#pragma unroll
    for (int k = 0; k < MAXK; ++k) {
        ids[k] = -1;
        if (k < K && t < T) ids[k] = topk_idx[static_cast<size_t>(t) * K + k];
    }
    bool bad = false;
    __syncwarp();
#pragma unroll
    for (int k = 0; k < MAXK; ++k) {
        if (k < K && t < T) {
            if (slot_valid(ids, k, E)) {
                // planes == 1: one mask per expert; planes == K: one per slot
                // index (slot-major capacity priority), plane k holding the
                // k-th choices
                atomicOr(&sm[(planes == 1 ? 0 : k) * E + ids[k]], 1u << lane);
            } else {
                bad = true;
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_device_status(status, MOE_DEV_BAD_ROUTING);
    __syncwarp();
    for (int i = lane; i < words; i += 32) {
        const int pl = i / E, j = i - pl * E;
        bitmap[(static_cast<size_t>(pl) * t_words + w) * E + j] = sm[i];
    }
}

// One block of 1024 threads.  Thread (p, j) = (tid / E, tid % E): expert j,
// word slice p of P = 1024 / E (consecutive threads read consecutive experts
// of one word: coalesced).  Per thread: the popcounts of its slice (up to
// SCAN_CACHE words loaded all at once and kept in registers for the second
// pass; longer slices -- many slot planes -- are read in batches of eight,
// twice); a scan over the slices of each expert; the per-word prefixes
// written; and an exclusive scan of kept over the experts for the offsets.
constexpr int SCAN_CACHE = 32;

// With bal.f non-null the block then computes the balance statistics of the
// batch as well (balance_block: the same arithmetic as the balance kernel),
// which saves moe_layer_forward that kernel.
__global__ void __launch_bounds__(1024)
scan_kernel(const uint32_t* __restrict__ bitmap, int E, int n_words, int capacity,
            int32_t* __restrict__ word_base, int32_t* __restrict__ counts,
            int32_t* __restrict__ kept, int32_t* __restrict__ offsets, BalanceArgs bal) {
    __shared__ int part[1024];
    __shared__ int kept_s[256];
    pdl_wait();
    pdl_allow_next();
    const int tid = threadIdx.x;
    const int P = 1024 / E;                                // >= 4: E <= 256
    const int p = tid / E, j = tid - p * E;
    const bool act = p < P;
    const int wpp = (n_words + P - 1) / P;
    const int w0 = act ? min(n_words, p * wpp) : 0;
    const int w1 = act ? min(n_words, w0 + wpp) : 0;
    const bool cached = wpp <= SCAN_CACHE;
    int pc[SCAN_CACHE];
    int sum = 0;
    if (cached) {
#pragma unroll
        for (int u = 0; u < SCAN_CACHE; ++u)
            pc[u] = (w0 + u < w1) ? __popc(__ldg(bitmap + static_cast<size_t>(w0 + u) * E + j)) : 0;
#pragma unroll
        for (int u = 0; u < SCAN_CACHE; ++u) sum += pc[u];
    } else {
        int w = w0;
        for (; w + 8 <= w1; w += 8) {
            uint32_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldg(bitmap + static_cast<size_t>(w + u) * E + j);
#pragma unroll
            for (int u = 0; u < 8; ++u) sum += __popc(v[u]);
        }
        for (; w < w1; ++w) sum += __popc(__ldg(bitmap + static_cast<size_t>(w) * E + j));
    }
    part[tid] = sum;
    __syncthreads();
    for (int off = 1; off < P; off <<= 1) {                // inclusive scan over the slices of j
        const int add = (act && p >= off) ? part[tid - off * E] : 0;
        __syncthreads();
        part[tid] += add;
        __syncthreads();
    }
    if (act && p == P - 1) {
        counts[j] = part[tid];
        kept_s[j] = capacity >= 0 ? min(part[tid], capacity) : part[tid];
    }
    {
        int run = part[tid] - sum;                         // words of j before this slice
        if (cached) {
#pragma unroll
            for (int u = 0; u < SCAN_CACHE; ++u) {
                if (w0 + u < w1) word_base[static_cast<size_t>(w0 + u) * E + j] = run;
                run += pc[u];
            }
        } else {
            int w = w0;
            for (; w + 8 <= w1; w += 8) {
                uint32_t v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = __ldg(bitmap + static_cast<size_t>(w + u) * E + j);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    word_base[static_cast<size_t>(w + u) * E + j] = run;
                    run += __popc(v[u]);
                }
            }
            for (; w < w1; ++w) {
                word_base[static_cast<size_t>(w) * E + j] = run;
                run += __popc(__ldg(bitmap + static_cast<size_t>(w) * E + j));
            }
        }
    }
    __syncthreads();
    const int kv = tid < E ? kept_s[tid] : 0;
    int incl = kv;
    for (int off = 1; off < E; off <<= 1) {                // inclusive scan of kept over experts
        const int add = (tid < E && tid >= off) ? kept_s[tid - off] : 0;
        __syncthreads();
        if (tid < E) kept_s[tid] = (incl += add);
        __syncthreads();
    }
    if (tid < E) {
        kept[tid] = kv;
        offsets[tid] = incl - kv;
        if (tid == E - 1) offsets[E] = incl;
    }
    if (bal.f != nullptr) {
        __syncthreads();                                   // counts written, kept_s and part free
        balance_block(counts, bal.psum, bal.blocks, bal.T, E, bal.K, bal.alpha, bal.f, bal.P, bal.loss,
                      reinterpret_cast<float*>(part), reinterpret_cast<float*>(kept_s));
    }
}

constexpr int SC_WARPS = 8;       // warps per scatter block

// W warps per token (W = 1 for large batches; up to 32 -- four blocks -- when
// there are too few tokens to fill the GPU); global warp g serves token g / W,
// share g % W.  Lanes 0..K-1 resolve the token's K slots to destination
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
    pdl_wait();
    pdl_allow_next();
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * SC_WARPS + (threadIdx.x >> 5);
    const int t = gw / wpt;
    const int sub = gw % wpt;                              // this warp's share of the row
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
                            int32_t* status, cudaStream_t st, const BalanceArgs* bal) {
    // warps per block: up to 8, with at most 32 KB of masks in shared memory
    const int words = dm.planes * dm.E;
    int wpb = 8;
    while (wpb > 1 && wpb * words * 4 > 32 * 1024) wpb >>= 1;
    cudaError_t e = launch_pdl(bitmap_kernel, dim3((dm.t_words + wpb - 1) / wpb), dim3(32 * wpb),
                               static_cast<size_t>(wpb) * words * 4, st, 1,
                               topk_idx, dm.T, dm.E, dm.K, dm.t_words, dm.planes, bitmap, status);
    if (e != cudaSuccess) return e;
    // the scan runs over the (plane, word) sequence: token order within a
    // plane, planes in slot order
    BalanceArgs none{};
    e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, st, 1, bitmap, dm.E, dm.planes * dm.t_words, dm.capacity,
                   word_base, counts, kept, offsets, bal ? *bal : none);
    if (e != cudaSuccess) return e;
    const int shared_copy = (dm.dtype == MOE_FP8_E4M3_BLOCK && dm.S > 0) ? 1 : 0;
    // warps per token: enough warps in flight to fill the GPU at small T
    int wpt = 1;
    while (wpt < 32 && static_cast<long long>(dm.T) * wpt < 148LL * 32) wpt *= 2;
    const int blocks = static_cast<int>((static_cast<long long>(dm.T) * wpt + SC_WARPS - 1) / SC_WARPS);
#define MOE_SCATTER(MODE) e = launch_pdl(scatter_kernel<MODE>, dim3(blocks), dim3(32 * SC_WARPS), 0, st, 1,        \
        x, topk_idx, bitmap, word_base, offsets, dm.T, dm.d, dm.E, dm.K, dm.capacity,                       \
        dm.r_cap, shared_copy, slot_row, row_slot, x_disp, x_disp_scales, wpt, dm.t_words, dm.slot_major)
    if (dm.dtype == MOE_F32) MOE_SCATTER(0);
    else if (dm.dtype == MOE_BF16) MOE_SCATTER(1);
    else MOE_SCATTER(2);
#undef MOE_SCATTER
    return e;
}

}  // namespace moe

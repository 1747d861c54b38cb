// Router logits on the tensor cores.
//
// "論文解説: DeepSeekMoE" §ルーティングとバランス損失: the router logits are
// W_r x with an fp32 router weight.  The activations x are exactly bf16, so
// the logits are computed as x (W_hi + W_mid + W_lo)^T where the three bf16
// planes are the successive roundings of W_r (8 + 8 + 8 significant bits, so
// their sum is W_r exactly): one bf16 GEMM with K = 3 d, each block of x
// multiplied by the same block of all three planes, into one fp32
// accumulator.
//
// router_split_kernel writes the planes side by side, W3 = [hi | mid | lo]
// (E rows of 3 d).  router_tc_kernel is a single-tile tcgen05 GEMM per CTA:
// grid (m-tiles of 128 tokens, n-tiles of BN experts, K splits over the
// 64-column blocks of d), TMA into a ring of 128-byte-swizzled stages that
// each hold one x block and the three plane blocks it multiplies (x is read
// once, not once per plane), one thread issuing tcgen05.mma into tensor
// memory, four epilogue warps writing fp32 partial logits part[split][t][e].
// The splits are summed in a fixed order afterwards.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cstring>
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int RBM = 128;
constexpr int RTHREADS = 192;
constexpr uint64_t kRouterWaitNs = 2000000000ull;
constexpr uint64_t kRouterDrainNs = 200000000ull;

struct __align__(64) RouterTcParams {
    CUtensorMap a_map;   // x (T, d) bf16
    CUtensorMap b_map;   // W3 (E, 3 d) bf16
    int T, E, d, d_blocks, ksplit;
    float* part;         // (ksplit, T, E)
    int32_t* status;
    uint64_t timeout_ns;
};

// A stage: one 64-column block of x (RBM rows) and the same block of each of
// the three planes (BN rows each), 128 bytes per row.
template <int BN> struct RCfg {
    static constexpr int STAGES = BN == 256 ? 2 : (BN == 128 ? 3 : (BN == 64 ? 5 : 7));
    static constexpr int A_BYTES = RBM * 128;
    static constexpr int B_BYTES = BN * 128;                // one plane
    static constexpr int OFF_B = STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + STAGES * 3 * B_BYTES;
    static constexpr int N_BARS = 2 * STAGES + 2;          // full, empty, accf, drain
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int TOTAL = OFF_MISC + 16;
    static constexpr int ALLOC = TOTAL + 1024;
    static constexpr uint32_t TMEM_COLS = BN;               // 32..256, a power of two
};

// Row blockIdx.y of W_r, four columns per thread (d is a multiple of 64 and
// W_r 16-byte aligned): one 16-byte load, one 8-byte store per plane.
__global__ void __launch_bounds__(256)
router_split_kernel(const float* __restrict__ W_r, int d, __nv_bfloat16* __restrict__ w3) {
    pdl_wait();
    pdl_allow_next();
    const int j = blockIdx.y;
    const float4* src = reinterpret_cast<const float4*>(W_r + static_cast<size_t>(j) * d);
    __nv_bfloat16* row = w3 + static_cast<size_t>(j) * 3 * d;
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < d / 4; c += gridDim.x * blockDim.x) {
        const float4 w4 = __ldg(src + c);
        const float w[4] = {w4.x, w4.y, w4.z, w4.w};
        __nv_bfloat16 pl[3][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(w[q]);
            const float r1 = w[q] - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const float r2 = r1 - __bfloat162float(mid);
            pl[0][q] = hi;
            pl[1][q] = mid;
            pl[2][q] = __float2bfloat16_rn(r2);
        }
#pragma unroll
        for (int p = 0; p < 3; ++p)
            *reinterpret_cast<uint2*>(row + static_cast<size_t>(p) * d + 4 * c) =
                *reinterpret_cast<const uint2*>(pl[p]);
    }
}

__device__ __forceinline__ bool warp_wait_r(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                            int32_t* status, uint64_t timeout_ns, int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(bar, parity, abort_flag, status, timeout_ns) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

template <int BN>
__global__ void __launch_bounds__(RTHREADS, 1)
router_tc_kernel(const __grid_constant__ RouterTcParams p) {
    using C = RCfg<BN>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* accf = empty + STAGES;
    uint64_t* drain = accf + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * RBM;
    const int n0 = blockIdx.y * BN;
    const int ks = blockIdx.z;
    const int kb_lo = static_cast<int>(static_cast<long long>(ks) * p.d_blocks / p.ksplit);
    const int kb_hi = static_cast<int>(static_cast<long long>(ks + 1) * p.d_blocks / p.ksplit);

    if (warp == 0) tmem_alloc<C::TMEM_COLS>(tmem_slot);
    if (warp == 1 && lane == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) { tma_prefetch_desc(&p.a_map); tma_prefetch_desc(&p.b_map); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();
    pdl_allow_next();

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                mbar_arrive_expect_tx(&full[stage], C::A_BYTES + 3 * C::B_BYTES);
                tma_load_2d(smem + stage * C::A_BYTES, &p.a_map, &full[stage], kb * 64, m0);
#pragma unroll
                for (int pl = 0; pl < 3; ++pl)
                    tma_load_2d(smem + C::OFF_B + (stage * 3 + pl) * C::B_BYTES, &p.b_map, &full[stage],
                                pl * p.d + kb * 64, n0);
                ++issued;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) {
                int s = stage;
                uint32_t ph = phase;
                const int pending = issued < STAGES ? issued : STAGES;
                for (int i = 0; i < pending; ++i) {
                    if (--s < 0) { s = STAGES - 1; ph ^= 1u; }
                    volatile int no_abort = 0;
                    mbar_wait_bounded(&full[s], ph, &no_abort, nullptr, kRouterDrainNs);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc(1, RBM, BN);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued_any = false;
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint64_t adesc = smem_desc_k_sw128(smem + stage * C::A_BYTES);
#pragma unroll
                for (int pl = 0; pl < 3; ++pl) {
                    const uint64_t bdesc = smem_desc_k_sw128(smem + C::OFF_B + (stage * 3 + pl) * C::B_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_f16(tmem_base, adesc + 2 * k, bdesc + 2 * k, idesc,
                                 (kb > kb_lo || pl > 0 || k > 0) ? 1u : 0u);
                }
                issued_any = true;
                umma_commit(&empty[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (ok) {
                umma_commit(accf);
            } else if (issued_any) {
                umma_commit(drain);
                volatile int no_abort = 0;
                mbar_wait_bounded(drain, 0, &no_abort, nullptr, kRouterDrainNs);
            }
        }
        __syncwarp();
    } else {
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int t = m0 + r;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        if (warp_wait_r(accf, 0, abort_flag, p.status, p.timeout_ns, lane)) {
            tc_fence_after();
            float* dst = p.part + (static_cast<size_t>(ks) * p.T + t) * p.E + n0;
            const int n_valid = min(BN, p.E - n0);
            const bool vec = (p.E & 3) == 0;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(c * 32), v);
                tmem_ld_wait();
                if (t < p.T) {
                    if (vec && c * 32 + 32 <= n_valid) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            reinterpret_cast<float4*>(dst + c * 32)[q] =
                                make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c * 32 + j < n_valid) dst[c * 32 + j] = __uint_as_float(v[j]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc<C::TMEM_COLS>(tmem_base);
    }
}

// ---------------------------------------------------------------- CTA pairs
//
// With two or more 128-token tiles, clusters of two CTAs share every MMA
// (tcgen05.mma.cta_group::2, M = 256 tokens: each CTA holds its own 128 rows
// of x and BN/2 rows of each weight plane, and receives its 128 rows of the
// accumulator).  Per SM that halves the plane bytes a stage moves into shared
// memory -- three quarters of a stage at BN = 256 -- so a stage is 64 KB
// instead of 112 KB and three of them fit where two did: the kernel waits on
// L2 latency with more bytes in flight.  Both CTAs' TMA loads signal the
// first CTA's stage barrier, where the pair's single MMA-issuing thread
// waits; tcgen05.commit with a CTA mask releases a stage in both CTAs and
// announces the finished accumulator to both epilogues.  Plain TMA loads only.
template <int BN> struct RCfg2 {
    static constexpr int BH = BN / 2;                       // plane rows per CTA
    static constexpr int A_BYTES = RBM * 128;
    static constexpr int B_BYTES = BH * 128;                // one plane, this CTA's half
    static constexpr int STAGE_BYTES = A_BYTES + 3 * B_BYTES;
    static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 8 ? 8 : (200 * 1024) / STAGE_BYTES;
    static constexpr int OFF_B = STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + STAGES * 3 * B_BYTES;
    static constexpr int N_BARS = 2 * STAGES + 2;          // full, empty, accf, drain
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int TOTAL = OFF_MISC + 16;
    static constexpr int ALLOC = TOTAL + 1024;
    static constexpr uint32_t TMEM_COLS = BN;
};

template <int BN>
__global__ void __launch_bounds__(RTHREADS, 1)
router_tc2_kernel(const __grid_constant__ RouterTcParams p) {
    using C = RCfg2<BN>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* accf = empty + STAGES;
    uint64_t* drain = accf + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();          // 0: issues the MMAs of the pair
    const int m0 = (blockIdx.x >> 1) * 2 * RBM + static_cast<int>(rank) * RBM;
    const int n0 = blockIdx.y * BN;
    const int ks = blockIdx.z;
    const int kb_lo = static_cast<int>(static_cast<long long>(ks) * p.d_blocks / p.ksplit);
    const int kb_hi = static_cast<int>(static_cast<long long>(ks + 1) * p.d_blocks / p.ksplit);

    if (warp == 0) tmem_alloc_pair<C::TMEM_COLS>(tmem_slot);
    if (warp == 1 && lane == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) { tma_prefetch_desc(&p.a_map); tma_prefetch_desc(&p.b_map); }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                   // barriers of both CTAs initialised
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();
    pdl_allow_next();

    if (warp == 0) {
        // ================= TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
                if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
                tma_load_2d_pair(smem + stage * C::A_BYTES, &p.a_map, bar0, kb * 64, m0);
#pragma unroll
                for (int pl = 0; pl < 3; ++pl)
                    tma_load_2d_pair(smem + C::OFF_B + (stage * 3 + pl) * C::B_BYTES, &p.b_map, bar0,
                                     pl * p.d + kb * 64, n0 + static_cast<int>(rank) * C::BH);
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) {
                // unwinding: copies still in flight land within microseconds
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 100000ull) { }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================= MMA issuer (first CTA of the pair)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = make_idesc(1, 2 * RBM, BN);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued_any = false;
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint64_t adesc = smem_desc_k_sw128(smem + stage * C::A_BYTES);
#pragma unroll
                for (int pl = 0; pl < 3; ++pl) {
                    const uint64_t bdesc = smem_desc_k_sw128(smem + C::OFF_B + (stage * 3 + pl) * C::B_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_f16_pair(tmem_base, adesc + 2 * k, bdesc + 2 * k, idesc,
                                      (kb > kb_lo || pl > 0 || k > 0) ? 1u : 0u);
                }
                issued_any = true;
                umma_commit_pair(&empty[stage], 0x3);       // stage free in both CTAs
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (ok) {
                umma_commit_pair(accf, 0x3);                // accumulator ready in both CTAs
            } else if (issued_any) {
                umma_commit_pair(drain, 0x1);
                volatile int no_abort = 0;
                mbar_wait_bounded(drain, 0, &no_abort, nullptr, kRouterDrainNs);
            }
        }
        __syncwarp();
    } else {
        // ================= epilogue (both CTAs): this CTA's 128 rows
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int t = m0 + r;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        if (warp_wait_r(accf, 0, abort_flag, p.status, p.timeout_ns, lane)) {
            tc_fence_after();
            float* dst = p.part + (static_cast<size_t>(ks) * p.T + t) * p.E + n0;
            const int n_valid = min(BN, p.E - n0);
            const bool vec = (p.E & 3) == 0;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(c * 32), v);
                tmem_ld_wait_regs(v);
                if (t < p.T) {
                    if (vec && c * 32 + 32 <= n_valid) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            reinterpret_cast<float4*>(dst + c * 32)[q] =
                                make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c * 32 + j < n_valid) dst[c * 32 + j] = __uint_as_float(v[j]);
                    }
                }
            }
        }
    }
    // ---- teardown: both CTAs are done with tensor memory and with each
    // other's barriers before either frees or exits
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair<C::TMEM_COLS>(tmem_base);
    }
}

template <int BN>
cudaError_t launch_bn2(const RouterTcPlan& plan, const RouterTcParams& p, cudaStream_t st) {
    constexpr int smem = RCfg2<BN>::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(router_tc2_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(router_tc2_kernel<BN>, dim3(2 * ((plan.mt + 1) / 2), plan.nt, plan.ksplit), dim3(RTHREADS),
                      smem, st, 2, p);
}

template <int BN>
cudaError_t launch_bn(const Dims& dm, const RouterTcPlan& plan, const RouterTcParams& p, cudaStream_t st) {
    constexpr int smem = RCfg<BN>::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(router_tc_kernel<BN>, dim3(plan.mt, plan.nt, plan.ksplit), dim3(RTHREADS), smem, st, 1, p);
}

}  // namespace

RouterTcPlan router_tc_plan(const Dims& dm) {
    RouterTcPlan pl{};
    pl.mt = (dm.T + RBM - 1) / RBM;
    const int kb_total = dm.d / 64;          // 64-column blocks of d
    const int target = 148;                  // CTAs for one wave on a B200
    int ep = 32;
    while (ep < dm.E && ep < 256) ep *= 2;
    if (pl.mt >= 8 || ep <= 64) {
        pl.bn = ep;                          // one n-tile holds every expert
    } else {
        pl.bn = 64;                          // few tokens: split the experts too
    }
    pl.nt = (dm.E + pl.bn - 1) / pl.bn;
    // CTA pairs once there are two token tiles to pair (an odd last tile is
    // paired with a tile of zero rows past T) and the expert tile is at least
    // 128 wide
    // (the pair halves the plane bytes a CTA stages, which is what fills a
    // stage once the expert tile is 128 wide or more; with narrower tiles the
    // x block dominates and single CTAs measured faster)
    pl.pair = (pl.mt >= 2 && pl.bn >= 128) ? 1 : 0;
    const int ctas_per_split = (pl.pair ? 2 * ((pl.mt + 1) / 2) : pl.mt) * pl.nt;
    int ks = target / ctas_per_split;
    if (ks < 1) ks = 1;
    if (ks > kb_total / 2) ks = kb_total / 2 > 0 ? kb_total / 2 : 1;
    pl.ksplit = ks;
    return pl;
}

cudaError_t launch_router_tc(const Dims& dm, const RouterTcPlan& plan, const void* x, const float* W_r,
                             void* w3, float* part, int32_t* status, cudaStream_t st) {
    const int col_blocks = (dm.d / 4 + 255) / 256;
    cudaError_t e = launch_pdl(router_split_kernel, dim3(col_blocks, dm.E), dim3(256), 0, st, 1, W_r, dm.d,
                               static_cast<__nv_bfloat16*>(w3));
    if (e != cudaSuccess) return e;
    RouterTcParams p;
    std::memset(&p, 0, sizeof(p));
    if (!encode_tma_2d(&p.a_map, x, dm.T, dm.d, 2, RBM)) return cudaErrorInvalidValue;
    if (!encode_tma_2d(&p.b_map, w3, dm.E, 3 * dm.d, 2, plan.bn)) return cudaErrorInvalidValue;
    p.T = dm.T;
    p.E = dm.E;
    p.d = dm.d;
    p.d_blocks = dm.d / 64;
    p.ksplit = plan.ksplit;
    p.part = part;
    p.status = status;
    p.timeout_ns = kRouterWaitNs;
    if (plan.pair) {
        if (!encode_tma_2d(&p.b_map, w3, dm.E, 3 * dm.d, 2, plan.bn / 2)) return cudaErrorInvalidValue;
        return plan.bn == 128 ? launch_bn2<128>(plan, p, st) : launch_bn2<256>(plan, p, st);
    }
    switch (plan.bn) {
        case 32: return launch_bn<32>(dm, plan, p, st);
        case 64: return launch_bn<64>(dm, plan, p, st);
        case 128: return launch_bn<128>(dm, plan, p, st);
        default: return launch_bn<256>(dm, plan, p, st);
    }
}

}  // namespace moe

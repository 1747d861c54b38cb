// Grouped expert FFN GEMMs in bf16 on the 5th-generation tensor cores.
//
// "論文解説: DeepSeekMoE" §アルゴリズム: each expert is Linear(d, d_ff) + bias
// -> SiLU -> Linear(d_ff, d) + bias.
//
// One persistent kernel computes C = epilogue(A B^T + bias) over the ragged
// segment list of ffn_common.cuh (routed experts from the device-side
// dispatch offsets, then the shared experts), so the host never synchronises.
//
// Per CTA (320 threads, one CTA per SM):
//   warp 0      TMA producer: A tile (128 rows x 64 bf16) and B tile
//               (256 rows x 64 bf16), 128-byte swizzle, into a ring of 4
//               shared-memory stages guarded by full/empty mbarriers;
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M=128, N=256, K=16)
//               into tensor memory and frees each stage with tcgen05.commit;
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (thread = row; the
//               warps of a lane quadrant split the 256 columns in halves),
//               bias, SiLU, bf16 rounding and 16-byte stores.
// Two 256-column accumulators in tensor memory let the epilogue of tile i
// overlap the MMAs of tile i+1.  Rows of a tile past the end of its segment
// are computed (they belong to the next segment or read as zeros) and never
// stored.
//
// Every wait is bounded (common.cuh); on expiry the CTA drains its in-flight
// copies and MMAs, frees its tensor memory and exits, and the host sees
// MOE_DEV_TIMEOUT in the workspace status word.
#include "ffn_common.cuh"

namespace moe {
namespace {

using namespace ffn;

constexpr int NUM_THREADS = 320;
constexpr int EPI_THREADS = 256;
constexpr int BN = 256, BK = 64, STAGES = 4, ACC_BUFS = 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;    // 2 s per wait
constexpr uint64_t kDrainTimeoutNs = 200000000ull;    // 0.2 s while unwinding

struct Smem {
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
    // full[STAGES], empty[STAGES], accf[2], acce[2], drain
    static constexpr int N_BARS = 2 * STAGES + 2 * ACC_BUFS + 1;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;   // tmem addr, abort flag
    static constexpr int OFF_SEG = OFF_MISC + 16;
    static constexpr int TOTAL = OFF_SEG + SegTable::SEG_INTS * 4;
    static constexpr int ALLOC = TOTAL + 1024;               // slack for 1 KB alignment
};

__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_ffn_bf16_kernel(const __grid_constant__ TcParams p) {
    using L = Smem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* accf = bars + 2 * STAGES;
    uint64_t* acce = accf + ACC_BUFS;
    uint64_t* drain = acce + ACC_BUFS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    SegTable seg(reinterpret_cast<int*>(smem + L::OFF_SEG));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- prologue: TMEM, barriers, segment table
    if (warp == 0) tmem_alloc<TMEM_COLS>(tmem_slot);
    if (warp == 1 && lane == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < ACC_BUFS; ++i) { mbar_init(&accf[i], 1); mbar_init(&acce[i], EPI_THREADS); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int gi = 0; gi < 2; ++gi) {
            if (p.g[gi].n_mats > 0) { tma_prefetch_desc(&p.a_map[gi]); tma_prefetch_desc(&p.b_map[gi]); }
        }
    }
    pdl_wait();          // the segment table reads the dispatch offsets
    pdl_allow_next();
    const int nseg = build_seg_table<BN>(p, seg, NUM_THREADS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total_tiles = seg.start[nseg];

    if (warp == 0) {
        // ================= TMA producer
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile<BN, BK>(tile, p, seg, nseg);
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[stage], L::A_BYTES + L::B_BYTES);
                    tma_load_2d(smem + L::OFF_A + stage * L::A_BYTES, &p.a_map[ti.grp], &full[stage],
                                kb * BK, ti.a_row);
                    tma_load_3d(smem + L::OFF_B + stage * L::B_BYTES, &p.b_map[ti.grp], &full[stage],
                                kb * BK, ti.n0, ti.mat);
                    ++issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                // unwinding: let every copy still in flight land before the CTA exits
                int s = stage;
                uint32_t ph = phase;
                const int pending = issued < STAGES ? issued : STAGES;
                for (int i = 0; i < pending; ++i) {
                    if (--s < 0) { s = STAGES - 1; ph ^= 1u; }
                    volatile int no_abort = 0;
                    mbar_wait_bounded(&full[s], ph, &no_abort, nullptr, kDrainTimeoutNs);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================= MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc(1, BM, BN);
            int stage = 0, abuf = 0;
            uint32_t phase = 0, aphase = 0;
            bool ok = true, issued_any = false;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile<BN, BK>(tile, p, seg, nseg);
                if (!mbar_wait_bounded(&acce[abuf], aphase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * BN);
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_k_sw128(smem + L::OFF_A + stage * L::A_BYTES);
                    const uint64_t bdesc = smem_desc_k_sw128(smem + L::OFF_B + stage * L::B_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k)            // 4 x 32 bytes of K per stage
                        umma_f16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                    issued_any = true;
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&accf[abuf]);
                if (++abuf == ACC_BUFS) { abuf = 0; aphase ^= 1u; }
            }
            if (!ok && issued_any) {
                // unwinding: wait for the MMAs already issued before TMEM is freed
                umma_commit(drain);
                volatile int no_abort = 0;
                mbar_wait_bounded(drain, 0, &no_abort, nullptr, kDrainTimeoutNs);
            }
        }
        __syncwarp();
    } else {
        // ================= epilogue (warps 2..9; TMEM lane quadrant = warp % 4)
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;                 // which 128 of the 256 columns
        const int r_local = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        int abuf = 0;
        uint32_t aphase = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const TileInfo ti = decode_tile<BN, BK>(tile, p, seg, nseg);
            const GroupDev& g = p.g[ti.grp];
            const bool row_ok = r_local < ti.rows_left;
            const int n_valid = min(BN, g.N - ti.n0);
            if (!warp_wait(&accf[abuf], aphase, abort_flag, p.status, p.timeout_ns, lane)) break;
            tc_fence_after();
            __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(g.C) +
                                  static_cast<size_t>(ti.c_row + r_local) * g.N + ti.n0;
            const float* bias = g.bias + static_cast<size_t>(ti.mat) * g.N + ti.n0;
#pragma unroll 1
            for (int cc = 0; cc < 2; ++cc) {
                const int c0 = half * 4 + cc * 2;         // two 32-column chunks in flight
                uint32_t r[2][32];
                tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(abuf * BN + c0 * 32), r[0]);
                tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(abuf * BN + c0 * 32 + 32), r[1]);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c = c0 + u;
                    if (!row_ok || c * 32 >= n_valid) continue;
                    uint32_t packed[16];
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4) {
                        const float4 b4 = __ldg(reinterpret_cast<const float4*>(bias + c * 32) + j4);
                        float v0 = __uint_as_float(r[u][4 * j4 + 0]) + b4.x;
                        float v1 = __uint_as_float(r[u][4 * j4 + 1]) + b4.y;
                        float v2 = __uint_as_float(r[u][4 * j4 + 2]) + b4.z;
                        float v3 = __uint_as_float(r[u][4 * j4 + 3]) + b4.w;
                        if (p.silu) {
                            v0 = silu_fast(v0); v1 = silu_fast(v1); v2 = silu_fast(v2); v3 = silu_fast(v3);
                        }
                        __nv_bfloat162 h01 = __floats2bfloat162_rn(v0, v1);
                        __nv_bfloat162 h23 = __floats2bfloat162_rn(v2, v3);
                        packed[2 * j4] = *reinterpret_cast<uint32_t*>(&h01);
                        packed[2 * j4 + 1] = *reinterpret_cast<uint32_t*>(&h23);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(crow + c * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                }
            }
            tc_fence_before();
            mbar_arrive(&acce[abuf]);
            if (++abuf == ACC_BUFS) { abuf = 0; aphase ^= 1u; }
        }
    }

    // ---- teardown: every role is done with TMEM
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem_base);
    }
}

}  // namespace

cudaError_t launch_grouped_ffn_bf16(const Dims&, const GemmArgs& a, cudaStream_t st) {
    TcParams p;
    if (!fill_params(p, a, 2, BN, kWaitTimeoutNs)) return cudaErrorInvalidValue;
    constexpr int smem = Smem::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(grouped_ffn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(grouped_ffn_bf16_kernel, dim3(device_sm_count()), dim3(NUM_THREADS), smem, st, 1, p);
}

}  // namespace moe

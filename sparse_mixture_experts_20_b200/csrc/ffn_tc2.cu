// Grouped expert FFN GEMMs in bf16 on CTA pairs (tcgen05 cta_group::2).
//
// "論文解説: DeepSeekMoE" §アルゴリズム: each expert is Linear(d, d_ff) + bias
// -> SiLU -> Linear(d_ff, d) + bias.
//
// Same computation and segment list as ffn_tc.cu, but two CTAs (a cluster of
// two SMs) share every MMA: one tcgen05.mma.cta_group::2 instruction computes
// a 256 x 256 x 16 block, with A rows 0..127 in the first CTA's shared memory
// and rows 128..255 in the second's, and weight rows split the same way.  Per
// SM that halves the weight bytes moved into shared memory and the number of
// MMA instructions issued.  A stage holds 128 columns of K (two 128-byte
// swizzle atoms, 64 KB per CTA) and the ring 3 stages.
//
// A scheduled tile is a pair of 128-row m-tiles of one segment and one
// 256-wide n-tile; when a segment has an odd number of m-tiles its last one
// runs alone as an M = 128 pair MMA (64 rows per CTA), so no MMA work is spent
// on a whole empty m-tile.  Each CTA loads its own A rows and its half of the
// weight rows; both TMA loads signal the first CTA's stage barrier, where the
// single MMA-issuing thread of the pair waits.  tcgen05.commit with a CTA
// mask releases the stage in both CTAs and announces a finished accumulator
// to both epilogues; each epilogue reads its own 128 accumulator rows and
// reports back to the first CTA.
//
// Per CTA (320 threads, one CTA per SM): warp 0 TMA producer, warp 1 MMA
// issuer (first CTA of the pair only), warps 2..9 epilogue (two warps per
// tensor-memory lane quadrant, 128 columns each; output chunks of 32 x 32
// leave through a 2 KB staging buffer per warp and TMA stores, which
// measured 5 % faster than per-thread row stores on the DeepSeekMoE-style
// layer, whose short K makes the epilogue a larger share of a tile).  Every wait is bounded
// (common.cuh).
#include <cstdlib>
#include "ffn_common.cuh"

namespace moe {
namespace {

using namespace ffn;

constexpr int NUM_THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr int BN = 256;            // weight rows per pair tile (128 per CTA)
constexpr int BN_HALF = BN / 2;
constexpr int SUB = 2;                 // 128-byte swizzle atoms of K per stage
constexpr int BK = 64 * SUB, STAGES = 3, ACC_BUFS = 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
constexpr uint64_t kDrainTimeoutNs = 200000000ull;

struct Smem {
    static constexpr int A_SUB = BM * 128;          // 128 rows x 64 bf16 (one swizzle atom of K)
    static constexpr int B_SUB = BN_HALF * 128;     // 128 weight rows x 64 bf16
    static constexpr int A_BYTES = SUB * A_SUB;
    static constexpr int B_BYTES = SUB * B_SUB;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
    // full[STAGES], empty[STAGES], accf[2], acce[2], drain
    static constexpr int N_BARS = 2 * STAGES + 2 * ACC_BUFS + 1;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int OFF_SEG = OFF_MISC + 16;
    // per epilogue warp one 2 KB staging buffer: a TMA store box of 32 rows x
    // 32 bf16 columns in the 64-byte swizzle
    static constexpr int OFF_STAGE = (OFF_SEG + SegTable::SEG_INTS * 4 + 1023) & ~1023;
    static constexpr int STAGE_BUF = 32 * 64;
    static constexpr int TOTAL = OFF_STAGE + EPI_WARPS * STAGE_BUF;
    static constexpr int ALLOC = TOTAL + 1024;
};

// Tile `tile` for CTA `rank` of the pair (a last n-tile with at most 128
// valid columns runs as an N = 128 pair MMA, 64 weight rows per CTA).  A
// segment of r rows has
// ceil(r / 128) m-tiles, scheduled two at a time (M = 256: 128 rows per CTA).
// An odd last m-tile is scheduled alone as an M = 128 pair MMA: 64 rows per
// CTA, whose accumulator uses 128 tensor-memory columns: lanes 0..63 hold
// output columns 0..127 of the 64 rows, lanes 64..127 columns 128..255 of the
// same rows.
struct PairTile {
    TileInfo ti;
    bool m128;
    bool n128;      // last n-tile with at most 128 valid columns: an N = 128 MMA
};

__device__ __forceinline__ PairTile decode_pair(int tile, const TcParams& p, const SegTable& t, int nseg, int rank) {
    int lo = 0, hi = nseg - 1;                      // last s with start[s] <= tile
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (t.start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int s = lo;
    const int local = tile - t.start[s];
    const int mtiles = ceil_div(t.rows[s], BM);
    const int mgroups = ceil_div(mtiles, 2);
    const int nt = local / mgroups, g = local % mgroups;
    PairTile pt;
    pt.m128 = (2 * g + 1 == mtiles);
    const int off = g * 2 * BM + rank * (pt.m128 ? BM / 2 : BM);
    pt.ti.grp = t.mat[s] >> 16;
    pt.ti.mat = t.mat[s] & 0xFFFF;
    pt.ti.rows_left = t.rows[s] - off;
    pt.ti.a_row = t.arow[s] + off;
    pt.ti.c_row = t.crow[s] + off;
    pt.ti.n0 = nt * BN;
    pt.ti.kblocks = ceil_div(p.g[pt.ti.grp].K, BK);
    // (not combined with M = 128, whose accumulator layout folds N)
    pt.n128 = !pt.m128 && p.g[pt.ti.grp].N - pt.ti.n0 <= BN_HALF;
    return pt;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_ffn_bf16_pair_kernel(const __grid_constant__ TcParams p) {
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
    const uint32_t rank = cluster_ctarank();          // 0: issues the MMAs of the pair
    const int pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

    if (warp == 0) tmem_alloc_pair<TMEM_COLS>(tmem_slot);
    if (warp == 1 && lane == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < ACC_BUFS; ++i) { mbar_init(&accf[i], 1); mbar_init(&acce[i], 2 * EPI_WARPS); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int gi = 0; gi < 2; ++gi)
            if (p.g[gi].n_mats > 0) { tma_prefetch_desc(&p.a_map[gi]); tma_prefetch_desc(&p.b_map[gi]); }
    }
    pdl_wait();          // the segment table reads the dispatch offsets
    pdl_allow_next();
    const int nseg = build_seg_table<BN, 2>(p, seg, NUM_THREADS);
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                   // barriers of both CTAs initialised
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total_tiles = seg.start[nseg];

    if (warp == 0) {
        // ================= TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = pair_id; tile < total_tiles && ok; tile += n_pairs) {
                // an M = 128 tile loads 128 rows from its 64-row offset; the
                // MMA reads the first 64
                const PairTile pt = decode_pair(tile, p, seg, nseg, static_cast<int>(rank));
                const TileInfo& ti = pt.ti;
                // an N = 128 tile: each CTA holds 64 weight rows (the box reads 128)
                const int b_row = ti.n0 + static_cast<int>(rank) * (pt.n128 ? BN_HALF / 2 : BN_HALF);
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (L::A_BYTES + L::B_BYTES));
#pragma unroll
                    for (int s = 0; s < SUB; ++s) {
                        // a K range past the end reads zeros (the MMA then adds nothing)
                        tma_load_2d_pair(smem + L::OFF_A + stage * L::A_BYTES + s * L::A_SUB, &p.a_map[ti.grp], bar0,
                                         kb * BK + s * 64, ti.a_row);
                        tma_load_3d_pair(smem + L::OFF_B + stage * L::B_BYTES + s * L::B_SUB, &p.b_map[ti.grp], bar0,
                                         kb * BK + s * 64, b_row, ti.mat);
                    }
                    ++issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                // unwinding: copies still in flight land within microseconds
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 100000ull) { }
            }
            (void)issued;
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================= MMA issuer (first CTA of the pair)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc256 = make_idesc(1, 2 * BM, BN);
            constexpr uint32_t idesc128 = make_idesc(1, BM, BN);
            constexpr uint32_t idesc256n = make_idesc(1, 2 * BM, BN_HALF);
            int stage = 0, abuf = 0;
            uint32_t phase = 0, aphase = 0;
            bool ok = true, issued_any = false;
            for (int tile = pair_id; tile < total_tiles && ok; tile += n_pairs) {
                const PairTile pt = decode_pair(tile, p, seg, nseg, 0);
                const TileInfo& ti = pt.ti;
                const uint32_t idesc = pt.m128 ? idesc128 : (pt.n128 ? idesc256n : idesc256);
                if (!mbar_wait_bounded(&acce[abuf], aphase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * BN);
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < SUB; ++s) {
                        const uint64_t adesc = smem_desc_k_sw128(smem + L::OFF_A + stage * L::A_BYTES + s * L::A_SUB);
                        const uint64_t bdesc = smem_desc_k_sw128(smem + L::OFF_B + stage * L::B_BYTES + s * L::B_SUB);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            umma_f16_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc,
                                          (kb > 0 || s > 0 || k > 0) ? 1u : 0u);
                    }
                    issued_any = true;
                    umma_commit_pair(&empty[stage], 0x3);   // stage free in both CTAs
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit_pair(&accf[abuf], 0x3);         // accumulator ready in both CTAs
                if (++abuf == ACC_BUFS) { abuf = 0; aphase ^= 1u; }
            }
            if (!ok && issued_any) {
                umma_commit_pair(drain, 0x1);
                volatile int no_abort = 0;
                mbar_wait_bounded(drain, 0, &no_abort, nullptr, kDrainTimeoutNs);
            }
        }
        __syncwarp();
    } else {
        // ================= epilogue (warps 2..9, both CTAs)
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r_local = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        // A chunk of 32 rows x 32 columns whose rows all lie in the segment
        // leaves through the warp's staging buffer (16-byte chunk q of a row at
        // q ^ ((row >> 1) & 3): the box's 64-byte swizzle) and one TMA store;
        // the buffer is rewritten once that store has read it.  Rows past a
        // segment's end are stored by their threads.
        uint8_t* stg = smem + L::OFF_STAGE + (warp - 2) * L::STAGE_BUF;
        int abuf = 0;
        uint32_t aphase = 0;
        for (int tile = pair_id; tile < total_tiles; tile += n_pairs) {
            const PairTile pt = decode_pair(tile, p, seg, nseg, static_cast<int>(rank));
            const TileInfo& ti = pt.ti;
            const GroupDev& g = p.g[ti.grp];
            // M = 256: quadrant = 32 rows, warp half = 128 columns (4 chunks);
            // M = 128: quadrants 0, 1 = rows 0..63 of columns 0..127, quadrants
            // 2, 3 = the same rows of columns 128..255; warp half = 64 columns
            const int r_loc = pt.m128 ? (quad & 1) * 32 + lane : r_local;
            const int n_base = (pt.m128 && quad >= 2) ? 128 : 0;
            // (an N = 128 tile: 128 columns, 64 per warp half, like M = 128)
            const bool narrow = pt.m128 || pt.n128;
            const int chunk0 = narrow ? half * 2 : half * 4;
            const int n_iter = narrow ? 1 : 2;
            const bool row_ok = r_loc < ti.rows_left;
            const int r_row0 = pt.m128 ? (quad & 1) * 32 : quad * 32;   // the warp's first row
            const bool full_rows = ti.rows_left >= r_row0 + 32;            // warp-uniform
            const int n_valid = min(BN, g.N - ti.n0);
            if (!warp_wait(&accf[abuf], aphase, abort_flag, p.status, p.timeout_ns, lane)) break;
            tc_fence_after();
            __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(g.C) +
                                  static_cast<size_t>(ti.c_row + r_loc) * g.N + ti.n0;
            const float* bias = g.bias + static_cast<size_t>(ti.mat) * g.N + ti.n0;
#pragma unroll 1
            for (int cc = 0; cc < n_iter; ++cc) {
                const int c0 = chunk0 + cc * 2;
                uint32_t r[2][32];
                tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(abuf * BN + c0 * 32), r[0]);
                tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(abuf * BN + c0 * 32 + 32), r[1]);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int col = n_base + (c0 + u) * 32;     // output column within the tile
                    if (col >= n_valid) continue;                // warp-uniform
                    if (!full_rows && !row_ok) continue;
                    uint32_t packed[16];
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4) {
                        const float4 b4 = __ldg(reinterpret_cast<const float4*>(bias + col) + j4);
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
                    if (full_rows) {
                        if (lane == 0) bulk_wait_read<0>();
                        __syncwarp();
                        uint8_t* row = stg + lane * 64;
                        const int sw = (lane >> 1) & 3;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<uint4*>(row + ((q ^ sw) << 4)) =
                                make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&p.c_map[ti.grp], stg, ti.n0 + col, ti.c_row + r_row0);
                            bulk_commit();
                        }
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(crow + col);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acce[abuf]), 0));
            if (++abuf == ACC_BUFS) { abuf = 0; aphase ^= 1u; }
        }
        // the stores have read their buffers and landed before the CTA exits
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    // ---- teardown: both CTAs are done with tensor memory and with each
    // other's barriers before either frees or exits
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair<TMEM_COLS>(tmem_base);
    }
}

}  // namespace

bool gemm_pairs_enabled() {
    static int enabled = -1;
    if (enabled < 0) {
        const char* v = std::getenv("MOE_GEMM_PAIR");
        enabled = (v && v[0] == '0') ? 0 : 1;
    }
    return enabled == 1;
}

cudaError_t launch_grouped_ffn_bf16_pair(const Dims&, const GemmArgs& a, cudaStream_t st) {
    TcParams p;
    if (!fill_params(p, a, 2, BN_HALF, kWaitTimeoutNs, 2)) return cudaErrorInvalidValue;
    constexpr int smem = Smem::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(grouped_ffn_bf16_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent: as many pairs as fit on the device at once
    int clusters = 0;
    cfg.gridDim = dim3(device_sm_count() & ~1);
    e = cudaOccupancyMaxActiveClusters(&clusters, grouped_ffn_bf16_pair_kernel, &cfg);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorLaunchOutOfResources;
    return launch_pdl(grouped_ffn_bf16_pair_kernel, dim3(2 * clusters), dim3(NUM_THREADS), smem, st, 2, p);
}

}  // namespace moe

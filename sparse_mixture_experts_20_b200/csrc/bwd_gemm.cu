// Grouped GEMMs of the layer backward in bf16 on the 5th-generation tensor
// cores: the recompute of z = x W1^T + b1, the two data-gradient GEMMs
// (dh = dy W2, dx = dz W1) and the two weight-gradient GEMMs (dW2 = dy^T
// SiLU(z), dW1 = dz^T x) of every routed and shared expert, plus the
// router's own gradients (dW_r = dl^T x, dl W_r).
//
// The forward these differentiate is "論文解説: DeepSeekMoE" §アルゴリズム (each
// expert Linear(d, d_ff) + bias -> SiLU -> Linear(d_ff, d) + bias) and
// §共有エキスパート機構 (routed experts on their tokens, shared experts on all).
//
// Two tile schedules over the same warp-specialised engine:
//   M-ragged  C[rows of a segment, N] = A[rows, K] * op(B_mat): the segment
//             rows are an expert's dispatched rows (device-side offsets, the
//             backward pads each expert's row count to a multiple of 16) or a
//             fixed count (the T tokens for a shared expert); K is fixed.
//   K-ragged  C_mat[M, N] = A[K rows, M]^T * B[K rows, N]: the contraction
//             runs over the segment's rows (weight gradients), so K differs
//             per matrix and is zero for an expert no token reached (the
//             output is then written as zeros).
// Operands are bf16 tiles staged by TMA in the 128-byte-swizzled layout; an
// operand whose contiguous dimension is M or N (a weight read transposed, or
// the activations of a weight gradient) is loaded as boxes of 64 elements of
// M/N by 64 rows of K and handed to tcgen05.mma as an MN-major operand
// (instruction descriptor transpose bits; shared-memory descriptor with the
// 64-element blocks LBO bytes apart and 8-row groups 1024 bytes apart).
//
// CTA pairs (clusters of two SMs, tcgen05 cta_group::2): one MMA instruction
// computes a 256 x 256 x 16 block with A rows 0..127 in the first CTA's
// shared memory and 128..255 in the second's, and the 256 output columns'
// B operand split the same way, so each SM stages half the B bytes of a
// single-CTA 128 x 256 tile.  A scheduled tile is two 128-row m-tiles and
// one 256-wide n-tile; an odd last m-tile runs as an M = 128 pair MMA (64
// rows per CTA; its accumulator folds the columns: lanes 0..63 hold columns
// 0..127, lanes 64..127 columns 128..255), a last n-tile with at most 128
// valid columns as an N = 128 pair MMA.  Both CTAs' TMA loads signal the
// first CTA's stage barrier, where the pair's single MMA-issuing thread
// waits; tcgen05.commit with a CTA mask frees the stage in both CTAs and
// hands a finished accumulator to both epilogues.
//
// Per CTA (320 threads, one CTA per SM): warp 0 TMA producer (ring of 6
// stages of 16 KB A + 16 KB B, paid for by one 2 KB output staging buffer per
// epilogue warp), warp 1 MMA issuer (first CTA of the pair),
// warps 2..9 epilogue (two warps per tensor-memory lane quadrant).
// Epilogues:
//   SILU_PAIR  v = acc + bias: SiLU(v) and SiLU'(v) as bf16 (recompute);
//   DSILU      acc * SiLU'(z) read from the recompute's output, as bf16 (dz);
//   F32        acc as fp32 (dx rows, weight gradients), or bf16 for dx rows
//              when the group asks for it.
// Output chunks of 32 rows x 32 columns (two boxes of 16 columns for fp32)
// leave through shared memory and TMA bulk stores (per-thread stores of a thread's 128-byte fp32 row pieces kept
// the weight-gradient kernel waiting on its store queue); rows past a
// segment's end are stored one by one.
// K is consumed in 16-row steps: a K-ragged segment issues only the steps
// inside its (16-padded) row count, so rows of the next segment that share
// the last TMA box are never multiplied.  Every wait is bounded (2 s); on
// expiry the CTA stops, the MMA thread waits for its issued MMAs, tensor
// memory is freed and MOE_DEV_TIMEOUT is left in the status word.
#include <cuda.h>
#include <cstring>
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;                 // rows of A per CTA (M = 256 per pair)
constexpr int BN = 256, BN_HALF = 128;  // output columns per pair tile, B rows/columns per CTA
constexpr int BK = 64, STAGES = 6, ACC_BUFS = 2;
constexpr int NUM_THREADS = 320, EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_SEGS = 256 + 8;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
constexpr uint64_t kDrainTimeoutNs = 200000000ull;
constexpr int BOX_BYTES = 64 * 64 * 2;  // one MN-major box: 64 elements x 64 K rows

enum Mode { MODE_RECOMP = 0, MODE_DSILU = 1, MODE_DX = 2, MODE_WGRAD = 3 };

template <int MODE> struct ModeTraits {
    static constexpr bool krag = MODE == MODE_WGRAD;
    static constexpr bool a_mn = MODE == MODE_WGRAD;
    static constexpr bool b_mn = MODE != MODE_RECOMP;
};

struct GroupDev {
    int n_mats;
    const int32_t* seg;
    int fixed;
    int M, N, K;
    int a_row_base, a_mat_stride;
    int b_col_stride, b_z_mat;
    const float* bias;
    const __nv_bfloat16* aux;
    void* out0;
    void* out1;
    int c_row_base, c_mat_rows, c_col_stride, ldc;
    long long c_mat_elems;
    int out_bf16;
};

struct __align__(64) Params {
    CUtensorMap a_map[2];
    CUtensorMap b_map[2];
    CUtensorMap c_map[2][2];       // outputs out0 / out1 of each group, for TMA stores
    GroupDev g[2];
    int tiles0, tiles_total;       // K-ragged schedule (host-known)
    int32_t* status;
    uint64_t timeout_ns;
};

struct Smem {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN_HALF * BK * 2;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    // per epilogue warp one 2 KB staging buffer: one TMA store box of 32 rows
    // x 64 bytes in the 64-byte swizzle (32 bf16 or 16 fp32 columns)
    static constexpr int STG_BYTES = 2048;
    static constexpr int STG_BUFS = 1;
    static constexpr int OFF_STAGE = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_BAR = OFF_STAGE + EPI_WARPS * STG_BUFS * STG_BYTES;
    static constexpr int N_BARS = 2 * STAGES + 2 * ACC_BUFS + 1;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int OFF_SEG = OFF_MISC + 16;
    static constexpr int SEG_INTS = (MAX_SEGS + 1) + 5 * MAX_SEGS;
    static constexpr int TOTAL = OFF_SEG + SEG_INTS * 4;
    static constexpr int ALLOC = TOTAL + 1024;
};
static_assert(Smem::A_BYTES == 2 * BOX_BYTES && Smem::B_BYTES == 2 * BOX_BYTES, "box layout");
static_assert(Smem::OFF_B % 1024 == 0 && Smem::A_BYTES % 1024 == 0 && Smem::B_BYTES % 1024 == 0,
              "stages start on 1024-byte swizzle atoms");
static_assert(Smem::OFF_STAGE % 1024 == 0 && Smem::STG_BYTES % 1024 == 0,
              "staging boxes start on 1024-byte swizzle atoms");
static_assert(Smem::ALLOC <= 227 * 1024, "shared memory budget");

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzled
// layout: 64-element (128-byte) rows of one K index, 8-row groups 1024 bytes
// apart (stride byte offset), consecutive 64-element blocks of M/N lbo bytes
// apart (leading byte offset); version 1 (bits 46-47), SWIZZLE_128B (61-63).
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(const void* tile, uint32_t lbo) {
    const uint32_t addr = smem_u32(tile);
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// M-ragged segment table (shared memory); a segment's tiles are its pairs of
// m-tiles times its n-tiles.
struct SegTable {
    int* start;   // first tile of each segment; start[nseg] = total
    int* rows;
    int* arow;
    int* crow;
    int* ccol;
    int* mat;     // group << 16 | matrix
    __device__ explicit SegTable(int* b)
        : start(b), rows(b + MAX_SEGS + 1), arow(rows + MAX_SEGS), crow(arow + MAX_SEGS),
          ccol(crow + MAX_SEGS), mat(ccol + MAX_SEGS) {}
};

__device__ int build_seg_table(const Params& p, SegTable& t) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n0 = p.g[0].n_mats, nseg = n0 + p.g[1].n_mats;
    for (int s = tid; s < nseg; s += NUM_THREADS) {
        const int gi = s < n0 ? 0 : 1;
        const int i = s - (gi ? n0 : 0);
        const GroupDev& g = p.g[gi];
        int rows, lo;
        if (g.seg) { lo = g.seg[i]; rows = g.seg[i + 1] - lo; }
        else { lo = 0; rows = g.fixed; }
        t.rows[s] = rows;
        t.arow[s] = g.a_row_base + (g.seg ? lo : i * g.a_mat_stride);
        t.crow[s] = g.c_row_base + (g.seg ? lo : i * g.c_mat_rows);
        t.ccol[s] = i * g.c_col_stride;
        t.mat[s] = (gi << 16) | i;
        t.start[s + 1] = cdiv(cdiv(rows, BM), 2) * cdiv(g.N, BN);
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < nseg; base += 32) {
            const int i = base + lane;
            int v = i < nseg ? t.start[i + 1] : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, v, off);
                if (lane >= off) v += o;
            }
            if (i < nseg) t.start[i + 1] = v + carry;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) t.start[0] = 0;
    }
    return nseg;
}

// One pair tile as seen by CTA `rank`.
struct Tile {
    int grp, mat;
    bool m128;       // odd last m-tile: an M = 128 pair MMA, 64 rows per CTA
    bool n128;       // last n-tile with at most 128 valid columns: an N = 128 pair MMA
    int m0;          // K-ragged: this CTA's first output row (of M)
    int rows_ok;     // valid output rows of this CTA (<= 128, <= 64 with m128)
    int a_row;       // M-ragged: this CTA's first A row; K-ragged: first K row (A and B)
    int n0;          // first output column of the pair tile
    int ksteps, kblocks;
    long long c_off; // element offset of this CTA's (row 0, column n0) in out0 / out1 / aux
    int ldc;
    int crow, ccol;  // the same as coordinates of the output's 2-D tensor map
};

template <bool KRAG>
__device__ __forceinline__ Tile decode(int tile, const Params& p, const SegTable& t, int nseg, int rank) {
    Tile ti;
    if constexpr (!KRAG) {
        int lo = 0, hi = nseg - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (t.start[mid] <= tile) lo = mid; else hi = mid - 1;
        }
        const int s = lo, local = tile - t.start[s];
        const int mt_n = cdiv(t.rows[s], BM), mg_n = cdiv(mt_n, 2);
        const int nt = local / mg_n, mg = local % mg_n;
        ti.grp = t.mat[s] >> 16;
        ti.mat = t.mat[s] & 0xFFFF;
        const GroupDev& g = p.g[ti.grp];
        ti.m128 = (2 * mg + 1 == mt_n);
        const int off = mg * 2 * BM + rank * (ti.m128 ? BM / 2 : BM);
        ti.m0 = 0;
        ti.rows_ok = min(ti.m128 ? BM / 2 : BM, t.rows[s] - off);
        ti.a_row = t.arow[s] + off;
        ti.n0 = nt * BN;
        ti.ksteps = g.K / 16;
        ti.ldc = g.ldc;
        ti.crow = t.crow[s] + off;
        ti.ccol = t.ccol[s] + ti.n0;
        ti.n128 = !ti.m128 && g.N - ti.n0 <= BN_HALF;
    } else {
        const int gi = tile >= p.tiles0 ? 1 : 0;
        const GroupDev& g = p.g[gi];
        const int local = tile - (gi ? p.tiles0 : 0);
        const int mt_n = cdiv(g.M, BM), mg_n = cdiv(mt_n, 2), nt_n = cdiv(g.N, BN);
        const int mat = local / (mg_n * nt_n), r = local % (mg_n * nt_n);
        const int nt = r / mg_n, mg = r % mg_n;
        ti.grp = gi;
        ti.mat = mat;
        ti.m128 = (2 * mg + 1 == mt_n);
        ti.m0 = mg * 2 * BM + rank * (ti.m128 ? BM / 2 : BM);
        ti.rows_ok = min(ti.m128 ? BM / 2 : BM, g.M - ti.m0);
        int lo, cnt;
        if (g.seg) { lo = g.seg[mat]; cnt = g.seg[mat + 1] - lo; }
        else { lo = mat * g.a_mat_stride; cnt = g.fixed; }
        ti.a_row = g.a_row_base + lo;
        ti.n0 = nt * BN;
        ti.ksteps = cdiv(cnt, 16);
        ti.ldc = g.ldc;
        ti.crow = mat * g.M + ti.m0;     // the matrices' outputs stacked as rows (c_mat_elems = M * ldc)
        ti.ccol = ti.n0;
        ti.n128 = !ti.m128 && g.N - ti.n0 <= BN_HALF;
    }
    ti.c_off = static_cast<long long>(ti.crow) * ti.ldc + ti.ccol;
    ti.kblocks = cdiv(ti.ksteps, 4);
    return ti;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, uint64_t timeout_ns, int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(bar, parity, abort_flag, status, timeout_ns) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ float dsilu_fast(float v) {
    const float sg = __fdividef(1.0f, 1.0f + __expf(-v));
    return sg * (1.0f + v * (1.0f - sg));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1) bwd_gemm_kernel(const __grid_constant__ Params p) {
    using L = Smem;
    using TR = ModeTraits<MODE>;
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
    pdl_wait();
    pdl_allow_next();
    int nseg = 0, total_tiles = p.tiles_total;
    if constexpr (!TR::krag) nseg = build_seg_table(p, seg);
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                   // barriers of both CTAs initialised
    tc_fence_after();
    if constexpr (!TR::krag) total_tiles = seg.start[nseg];
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ================= TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = pair_id; tile < total_tiles && ok; tile += n_pairs) {
                const Tile ti = decode<TR::krag>(tile, p, seg, nseg, static_cast<int>(rank));
                const GroupDev& g = p.g[ti.grp];
                const void* amap = &p.a_map[ti.grp];
                const void* bmap = &p.b_map[ti.grp];
                const int bz = g.b_z_mat ? ti.mat : 0;
                // this CTA's B rows (K-major) or columns (MN-major): half of
                // the pair's 256, or 64 of an N = 128 tile (whose box reads 128)
                const int bhalf = ti.n0 + static_cast<int>(rank) * (ti.n128 ? BN_HALF / 2 : BN_HALF);
                const int bcol = bhalf + (TR::krag ? ti.mat * g.b_col_stride : 0);
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (L::A_BYTES + L::B_BYTES));
                    uint8_t* sa = smem + L::OFF_A + stage * L::A_BYTES;
                    uint8_t* sb = smem + L::OFF_B + stage * L::B_BYTES;
                    const int k0 = kb * BK;
                    if constexpr (TR::a_mn) {
                        tma_load_2d_pair(sa, amap, bar0, ti.m0, ti.a_row + k0);
                        tma_load_2d_pair(sa + BOX_BYTES, amap, bar0, ti.m0 + 64, ti.a_row + k0);
                    } else {
                        tma_load_2d_pair(sa, amap, bar0, k0, ti.a_row);
                    }
                    if constexpr (TR::b_mn) {
                        const int krow = TR::krag ? ti.a_row + k0 : k0;
                        tma_load_3d_pair(sb, bmap, bar0, bcol, krow, bz);
                        tma_load_3d_pair(sb + BOX_BYTES, bmap, bar0, bcol + 64, krow, bz);
                    } else {
                        tma_load_3d_pair(sb, bmap, bar0, k0, bhalf, bz);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
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
            constexpr uint32_t tbits = (TR::a_mn ? (1u << 15) : 0u) | (TR::b_mn ? (1u << 16) : 0u);
            constexpr uint32_t idesc256 = make_idesc(1, 2 * BM, BN) | tbits;
            constexpr uint32_t idesc128 = make_idesc(1, BM, BN) | tbits;
            constexpr uint32_t idesc256n = make_idesc(1, 2 * BM, BN_HALF) | tbits;
            // K step of 16: 32 bytes along a K-major row, or 16 rows (2048
            // bytes) of an MN-major block; descriptor units of 16 B
            constexpr uint64_t a_step = TR::a_mn ? 128 : 2;
            constexpr uint64_t b_step = TR::b_mn ? 128 : 2;
            int stage = 0, abuf = 0;
            uint32_t phase = 0, aphase = 0;
            bool ok = true, issued_any = false;
            for (int tile = pair_id; tile < total_tiles && ok; tile += n_pairs) {
                const Tile ti = decode<TR::krag>(tile, p, seg, nseg, 0);
                const uint32_t idesc = ti.m128 ? idesc128 : (ti.n128 ? idesc256n : idesc256);
                if (!mbar_wait_bounded(&acce[abuf], aphase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * BN);
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint8_t* sa = smem + L::OFF_A + stage * L::A_BYTES;
                    const uint8_t* sb = smem + L::OFF_B + stage * L::B_BYTES;
                    const uint64_t adesc = TR::a_mn ? smem_desc_mn_sw128(sa, BOX_BYTES) : smem_desc_k_sw128(sa);
                    const uint64_t bdesc = TR::b_mn ? smem_desc_mn_sw128(sb, BOX_BYTES) : smem_desc_k_sw128(sb);
                    const int steps = min(4, ti.ksteps - kb * 4);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < steps)
                            umma_f16_pair(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc,
                                          (kb > 0 || k > 0) ? 1u : 0u);
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
        // ================= epilogue (warps 2..9, both CTAs; TMEM lane quadrant = warp % 4)
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        // A chunk of 32 rows x 32 columns whose rows all lie in the tile's
        // valid rows leaves through shared memory and TMA stores: the warp
        // writes 32 rows of 64 bytes into its staging buffer (16-byte chunk q
        // of a row at q ^ ((row >> 1) & 3): the box's 64-byte swizzle, which
        // also spreads the writes over the banks) and one lane stores the
        // box; fp32 chunks take two boxes.  The buffer is rewritten only after
        // the store issued from it has read it.  Other rows are stored by
        // their threads.
        uint8_t* stg = smem + L::OFF_STAGE + (warp - 2) * L::STG_BUFS * L::STG_BYTES;
        int sbuf = 0;
        auto stage_begin = [&]() -> uint8_t* {
            if (lane == 0) {
                if (L::STG_BUFS == 2) bulk_wait_read<1>();
                else bulk_wait_read<0>();
            }
            __syncwarp();
            return stg + sbuf * L::STG_BYTES;
        };
        auto stage_end = [&](const void* map, int x, int y) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(map, stg + sbuf * L::STG_BYTES, x, y);
                bulk_commit();
            }
            if (L::STG_BUFS == 2) sbuf ^= 1;
        };
        // one 64-byte row of a box: 16-byte chunk q at q ^ ((row >> 1) & 3)
        auto put_row64 = [&](uint8_t* buf, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                             uint32_t b1, uint32_t b2, uint32_t b3, uint32_t c0, uint32_t c1, uint32_t c2,
                             uint32_t c3, uint32_t d0, uint32_t d1, uint32_t d2, uint32_t d3) {
            uint8_t* row = buf + lane * 64;
            const int sw = (lane >> 1) & 3;
            *reinterpret_cast<uint4*>(row + ((0 ^ sw) << 4)) = make_uint4(a0, a1, a2, a3);
            *reinterpret_cast<uint4*>(row + ((1 ^ sw) << 4)) = make_uint4(b0, b1, b2, b3);
            *reinterpret_cast<uint4*>(row + ((2 ^ sw) << 4)) = make_uint4(c0, c1, c2, c3);
            *reinterpret_cast<uint4*>(row + ((3 ^ sw) << 4)) = make_uint4(d0, d1, d2, d3);
        };
        int abuf = 0;
        uint32_t aphase = 0;
        for (int tile = pair_id; tile < total_tiles; tile += n_pairs) {
            const Tile ti = decode<TR::krag>(tile, p, seg, nseg, static_cast<int>(rank));
            const GroupDev& g = p.g[ti.grp];
            // M = 256: quadrant = 32 rows, warp half = 128 columns (4 chunks);
            // M = 128: quadrants 0, 1 = rows 0..63 of columns 0..127,
            // quadrants 2, 3 = the same rows of columns 128..255, warp half =
            // 64 columns; N = 128: quadrant = 32 rows, warp half = 64 columns
            const int r_row0 = ti.m128 ? (quad & 1) * 32 : quad * 32;   // the warp's first row
            const int r_loc = r_row0 + lane;
            const int n_base = (ti.m128 && quad >= 2) ? BN_HALF : 0;
            const bool narrow = ti.m128 || ti.n128;
            const int chunk0 = narrow ? half * 2 : half * 4;
            const int n_iter = narrow ? 1 : 2;
            const bool row_ok = r_loc < ti.rows_ok;
            const bool full_rows = ti.rows_ok >= r_row0 + 32;            // warp-uniform
            const int n_valid = g.N - ti.n0;
            const bool f32_out = (MODE == MODE_WGRAD) || (MODE == MODE_DX && !g.out_bf16);
            if (!warp_wait(&accf[abuf], aphase, abort_flag, p.status, p.timeout_ns, lane)) break;
            tc_fence_after();
            const long long row_off = ti.c_off + static_cast<long long>(r_loc) * ti.ldc;
#pragma unroll 1
            for (int cc = 0; cc < n_iter; ++cc) {
                const int c0 = chunk0 + cc * 2;
                uint32_t r[2][32];
                if (ti.ksteps > 0) {
                    tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(abuf * BN + c0 * 32), r[0]);
                    tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(abuf * BN + c0 * 32 + 32), r[1]);
                    tmem_ld_wait_regs(r[0]);
                    tmem_ld_wait_regs(r[1]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) { r[0][i] = 0u; r[1][i] = 0u; }
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int col = n_base + (c0 + u) * 32;            // output column within the tile
                    if (col >= n_valid) continue;                      // warp-uniform
                    if (!full_rows && !row_ok) continue;
                    const long long off = row_off + col;
                    uint32_t o0[16], o1[16];                           // bf16 results, two per word
                    if constexpr (MODE == MODE_RECOMP) {
                        const float* bias = g.bias + static_cast<long long>(ti.mat) * g.N + ti.n0 + col;
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 b4 = __ldg(reinterpret_cast<const float4*>(bias) + j4);
                            const float v0 = __uint_as_float(r[u][4 * j4 + 0]) + b4.x;
                            const float v1 = __uint_as_float(r[u][4 * j4 + 1]) + b4.y;
                            const float v2 = __uint_as_float(r[u][4 * j4 + 2]) + b4.z;
                            const float v3 = __uint_as_float(r[u][4 * j4 + 3]) + b4.w;
                            o0[2 * j4] = pack_bf16x2(silu_fast(v0), silu_fast(v1));
                            o0[2 * j4 + 1] = pack_bf16x2(silu_fast(v2), silu_fast(v3));
                            o1[2 * j4] = pack_bf16x2(dsilu_fast(v0), dsilu_fast(v1));
                            o1[2 * j4 + 1] = pack_bf16x2(dsilu_fast(v2), dsilu_fast(v3));
                        }
                    } else if constexpr (MODE == MODE_DSILU) {
                        const uint4* sp = reinterpret_cast<const uint4*>(g.aux + off);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 s4 = __ldg(sp + q);
                            const uint32_t sw[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                            for (int w = 0; w < 4; ++w) {
                                const float2 sf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sw[w]));
                                const int j = 8 * q + 2 * w;
                                o0[4 * q + w] = pack_bf16x2(__uint_as_float(r[u][j]) * sf.x,
                                                            __uint_as_float(r[u][j + 1]) * sf.y);
                            }
                        }
                    } else {
#pragma unroll
                        for (int w = 0; w < 16; ++w)
                            o0[w] = pack_bf16x2(__uint_as_float(r[u][2 * w]), __uint_as_float(r[u][2 * w + 1]));
                    }
                    if (full_rows) {
                        const int x = ti.ccol + col, y = ti.crow + r_row0;
                        if (f32_out) {
                            // two boxes of 16 fp32 columns
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                const uint32_t* v = r[u] + 16 * hh;
                                put_row64(stage_begin(), v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7], v[8], v[9],
                                          v[10], v[11], v[12], v[13], v[14], v[15]);
                                stage_end(&p.c_map[ti.grp][0], x + 16 * hh, y);
                            }
                        } else {
                            put_row64(stage_begin(), o0[0], o0[1], o0[2], o0[3], o0[4], o0[5], o0[6], o0[7], o0[8],
                                      o0[9], o0[10], o0[11], o0[12], o0[13], o0[14], o0[15]);
                            stage_end(&p.c_map[ti.grp][0], x, y);
                            if constexpr (MODE == MODE_RECOMP) {
                                put_row64(stage_begin(), o1[0], o1[1], o1[2], o1[3], o1[4], o1[5], o1[6], o1[7],
                                          o1[8], o1[9], o1[10], o1[11], o1[12], o1[13], o1[14], o1[15]);
                                stage_end(&p.c_map[ti.grp][1], x, y);
                            }
                        }
                    } else if (f32_out) {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(g.out0) + off);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            dst[q] = make_float4(__uint_as_float(r[u][4 * q]), __uint_as_float(r[u][4 * q + 1]),
                                                 __uint_as_float(r[u][4 * q + 2]), __uint_as_float(r[u][4 * q + 3]));
                    } else {
                        uint4* d0 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out0) + off);
#pragma unroll
                        for (int q = 0; q < 4; ++q) d0[q] = make_uint4(o0[4 * q], o0[4 * q + 1], o0[4 * q + 2], o0[4 * q + 3]);
                        if constexpr (MODE == MODE_RECOMP) {
                            uint4* d1 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out1) + off);
#pragma unroll
                            for (int q = 0; q < 4; ++q) d1[q] = make_uint4(o1[4 * q], o1[4 * q + 1], o1[4 * q + 2], o1[4 * q + 3]);
                        }
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

// Host: device copy of a group and its tensor maps.
bool fill_group(Params& p, int gi, const BwdGemmGroup& h, bool a_mn, bool b_mn, bool krag, bool out_f32) {
    GroupDev& d = p.g[gi];
    d.n_mats = h.n_mats;
    if (h.n_mats == 0) return true;
    d.seg = h.seg;
    d.fixed = h.fixed;
    d.M = h.M;
    d.N = h.N;
    d.K = h.K;
    d.a_row_base = h.a_row_base;
    d.a_mat_stride = h.a_mat_stride;
    d.b_col_stride = h.b_col_stride;
    d.b_z_mat = h.b_z_mat;
    d.bias = h.bias;
    d.aux = static_cast<const __nv_bfloat16*>(h.aux);
    d.out0 = h.out0;
    d.out1 = h.out1;
    d.c_row_base = h.c_row_base;
    d.c_mat_rows = h.c_mat_rows;
    d.c_col_stride = h.c_col_stride;
    d.ldc = h.ldc;
    d.c_mat_elems = h.c_mat_elems;
    d.out_bf16 = h.out_bf16;
    // A (a_rows, a_cols): K-major boxes of 64 K x 128 rows, MN-major boxes of
    // 64 M x 64 K rows; B (b_mats, b_rows, b_cols): K-major boxes of 64 K x
    // 128 rows of N, MN-major boxes of 64 N x 64 rows of K
    if (!encode_tma_2d(&p.a_map[gi], h.A, h.a_rows, h.a_cols, 2, a_mn ? 64 : BM)) return false;
    if (!encode_tma_3d(&p.b_map[gi], h.B, h.b_mats, h.b_rows, h.b_cols, 2, b_mn ? 64 : BN_HALF)) return false;
    // outputs as 2-D (rows, ldc) tensors for 32 x 32 TMA store boxes; the
    // weight gradients' matrices stacked as rows
    const int rows = krag ? h.n_mats * h.M : h.c_rows;
    for (int o = 0; o < 2; ++o) {
        void* out = o == 0 ? h.out0 : h.out1;
        if (!out) continue;
        const bool ok = encode_tma_2d_store64(&p.c_map[gi][o], out, rows, h.ldc, out_f32 ? 4 : 2, 32);
        if (!ok) return false;
    }
    return true;
}

template <int MODE>
cudaError_t launch_mode(const BwdGemmArgs& a, cudaStream_t st) {
    using TR = ModeTraits<MODE>;
    Params p;
    std::memset(&p, 0, sizeof(p));
    for (int gi = 0; gi < 2; ++gi)
        if (!fill_group(p, gi, a.g[gi], TR::a_mn, TR::b_mn, TR::krag,
                        MODE == MODE_WGRAD || (MODE == MODE_DX && !a.g[gi].out_bf16)))
            return cudaErrorInvalidValue;
    int tiles[2] = {0, 0};
    for (int gi = 0; gi < 2; ++gi) {
        const BwdGemmGroup& g = a.g[gi];
        if (g.n_mats > 0 && TR::krag)
            tiles[gi] = g.n_mats * (((g.M + BM - 1) / BM + 1) / 2) * ((g.N + BN - 1) / BN);
    }
    p.tiles0 = tiles[0];
    p.tiles_total = tiles[0] + tiles[1];
    p.status = a.status;
    p.timeout_ns = kWaitTimeoutNs;
    constexpr int smem = Smem::ALLOC;
    cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // persistent: as many pairs as fit on the device at once
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(device_sm_count() & ~1);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, bwd_gemm_kernel<MODE>, &cfg);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorLaunchOutOfResources;
    return launch_pdl(bwd_gemm_kernel<MODE>, dim3(2 * clusters), dim3(NUM_THREADS), smem, st, 2, p);
}

}  // namespace

cudaError_t launch_bwd_gemm(BwdGemmKind kind, const BwdGemmArgs& a, cudaStream_t st) {
    if (a.g[0].n_mats + a.g[1].n_mats > MAX_SEGS) return cudaErrorInvalidValue;
    switch (kind) {
        case BWD_RECOMPUTE: return launch_mode<MODE_RECOMP>(a, st);
        case BWD_DGRAD_SILU: return launch_mode<MODE_DSILU>(a, st);
        case BWD_DGRAD_F32: return launch_mode<MODE_DX>(a, st);
        case BWD_WGRAD: return launch_mode<MODE_WGRAD>(a, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace moe

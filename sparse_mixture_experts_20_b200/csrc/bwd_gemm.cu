// Grouped GEMMs of the layer backward in bf16 on the 5th-generation tensor
// cores: the recompute of z = x W1^T + b1, the two data-gradient GEMMs
// (dh = dy W2, dx = dz W1) and the two weight-gradient GEMMs (dW2 = dy^T
// SiLU(z), dW1 = dz^T x) of every routed and shared expert.
//
// The forward these differentiate is "論文解説: DeepSeekMoE" §アルゴリズム (each
// expert Linear(d, d_ff) + bias -> SiLU -> Linear(d_ff, d) + bias) and
// §共有エキスパート機構 (routed experts on their tokens, shared experts on all).
//
// Two tile schedules over the same warp-specialised engine (320 threads, one
// CTA per SM, persistent):
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
// Roles: warp 0 TMA producer (ring of 4 stages of 16 KB A + 32 KB B), warp 1
// MMA issuer (M=128, N=256, K=16 per instruction, fp32 accumulators in
// tensor memory, two 256-column buffers), warps 2..9 epilogue (thread = row,
// two warps per lane quadrant split the 256 columns).  Epilogues:
//   SILU_PAIR  v = acc + bias: SiLU(v) and SiLU'(v) as bf16 (recompute);
//   DSILU      acc * SiLU'(z) read from the recompute's output, as bf16 (dz);
//   F32        acc as fp32 (dx rows, weight gradients), or bf16 for dx rows
//              when the group asks for it.
// K is consumed in 16-row steps: a K-ragged segment issues only the steps
// inside its (16-padded) row count, so rows of the next segment that share
// the last TMA box are never multiplied.  Every wait is bounded (2 s); on
// expiry the CTA drains its copies and MMAs, frees tensor memory, exits and
// leaves MOE_DEV_TIMEOUT in the status word.
#include <cuda.h>
#include <cstring>
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4, ACC_BUFS = 2;
constexpr int NUM_THREADS = 320, EPI_THREADS = 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_SEGS = 256 + 8;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
constexpr uint64_t kDrainTimeoutNs = 200000000ull;
constexpr int BOX_BYTES = 64 * 64 * 2;       // one MN-major box: 64 elements x 64 K rows

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
    GroupDev g[2];
    int tiles0, tiles_total;       // K-ragged schedule (host-known)
    int32_t* status;
    uint64_t timeout_ns;
};

struct Smem {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
    static constexpr int N_BARS = 2 * STAGES + 2 * ACC_BUFS + 1;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int OFF_SEG = OFF_MISC + 16;
    static constexpr int SEG_INTS = (MAX_SEGS + 1) + 5 * MAX_SEGS;
    static constexpr int TOTAL = OFF_SEG + SEG_INTS * 4;
    static constexpr int ALLOC = TOTAL + 1024;
};
static_assert(Smem::A_BYTES == 2 * BOX_BYTES && Smem::B_BYTES == 4 * BOX_BYTES, "box layout");
static_assert(Smem::OFF_B % 1024 == 0 && Smem::A_BYTES % 1024 == 0 && Smem::B_BYTES % 1024 == 0,
              "stages start on 1024-byte swizzle atoms");
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

// M-ragged segment table (shared memory).
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
        t.start[s + 1] = cdiv(rows, BM) * cdiv(g.N, BN);
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

struct Tile {
    int grp, mat;
    int m0;          // K-ragged: first output row (of M); M-ragged: 0
    int rows_ok;     // valid output rows of the tile (<= 128)
    int a_row;       // M-ragged: first A row; K-ragged: first K row (A and B)
    int n0;
    int ksteps, kblocks;
    long long c_off; // element offset of the tile's (row 0, column n0) in out0 / out1 / aux
    int ldc;
};

template <bool KRAG>
__device__ __forceinline__ Tile decode(int tile, const Params& p, const SegTable& t, int nseg) {
    Tile ti;
    if constexpr (!KRAG) {
        int lo = 0, hi = nseg - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (t.start[mid] <= tile) lo = mid; else hi = mid - 1;
        }
        const int s = lo, local = tile - t.start[s];
        const int mt_n = cdiv(t.rows[s], BM);
        const int nt = local / mt_n, mt = local % mt_n;
        ti.grp = t.mat[s] >> 16;
        ti.mat = t.mat[s] & 0xFFFF;
        const GroupDev& g = p.g[ti.grp];
        ti.m0 = 0;
        ti.rows_ok = min(BM, t.rows[s] - mt * BM);
        ti.a_row = t.arow[s] + mt * BM;
        ti.n0 = nt * BN;
        ti.ksteps = g.K / 16;
        ti.ldc = g.ldc;
        ti.c_off = static_cast<long long>(t.crow[s] + mt * BM) * g.ldc + t.ccol[s] + ti.n0;
    } else {
        const int gi = tile >= p.tiles0 ? 1 : 0;
        const GroupDev& g = p.g[gi];
        const int local = tile - (gi ? p.tiles0 : 0);
        const int mt_n = cdiv(g.M, BM), nt_n = cdiv(g.N, BN);
        const int mat = local / (mt_n * nt_n), r = local % (mt_n * nt_n);
        const int nt = r / mt_n, mt = r % mt_n;
        ti.grp = gi;
        ti.mat = mat;
        ti.m0 = mt * BM;
        ti.rows_ok = min(BM, g.M - ti.m0);
        int lo, cnt;
        if (g.seg) { lo = g.seg[mat]; cnt = g.seg[mat + 1] - lo; }
        else { lo = mat * g.a_mat_stride; cnt = g.fixed; }
        ti.a_row = g.a_row_base + lo;
        ti.n0 = nt * BN;
        ti.ksteps = cdiv(cnt, 16);
        ti.ldc = g.ldc;
        ti.c_off = static_cast<long long>(mat) * g.c_mat_elems + static_cast<long long>(ti.m0) * g.ldc + ti.n0;
    }
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

    if (warp == 0) tmem_alloc<TMEM_COLS>(tmem_slot);
    if (warp == 1 && lane == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < ACC_BUFS; ++i) { mbar_init(&accf[i], 1); mbar_init(&acce[i], EPI_THREADS); }
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
    tc_fence_after();
    if constexpr (!TR::krag) total_tiles = seg.start[nseg];
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ================= TMA producer
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const Tile ti = decode<TR::krag>(tile, p, seg, nseg);
                const GroupDev& g = p.g[ti.grp];
                const void* amap = &p.a_map[ti.grp];
                const void* bmap = &p.b_map[ti.grp];
                const int bz = g.b_z_mat ? ti.mat : 0;
                const int bcol = ti.n0 + (TR::krag ? ti.mat * g.b_col_stride : 0);
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[stage], L::A_BYTES + L::B_BYTES);
                    uint8_t* sa = smem + L::OFF_A + stage * L::A_BYTES;
                    uint8_t* sb = smem + L::OFF_B + stage * L::B_BYTES;
                    const int k0 = kb * BK;
                    if constexpr (TR::a_mn) {
                        tma_load_2d(sa, amap, &full[stage], ti.m0, ti.a_row + k0);
                        tma_load_2d(sa + BOX_BYTES, amap, &full[stage], ti.m0 + 64, ti.a_row + k0);
                    } else {
                        tma_load_2d(sa, amap, &full[stage], k0, ti.a_row);
                    }
                    if constexpr (TR::b_mn) {
                        const int krow = TR::krag ? ti.a_row + k0 : k0;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tma_load_3d(sb + j * BOX_BYTES, bmap, &full[stage], bcol + 64 * j, krow, bz);
                    } else {
                        tma_load_3d(sb, bmap, &full[stage], k0, ti.n0, bz);
                    }
                    ++issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
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
            constexpr uint32_t idesc = make_idesc(1, BM, BN) | (TR::a_mn ? (1u << 15) : 0u) |
                                       (TR::b_mn ? (1u << 16) : 0u);
            int stage = 0, abuf = 0;
            uint32_t phase = 0, aphase = 0;
            bool ok = true, issued_any = false;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const Tile ti = decode<TR::krag>(tile, p, seg, nseg);
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
                    // K step of 16: 32 bytes along a K-major row, or 16 rows
                    // (2048 bytes) of an MN-major block; descriptor units of 16 B
                    constexpr uint64_t a_step = TR::a_mn ? 128 : 2;
                    constexpr uint64_t b_step = TR::b_mn ? 128 : 2;
                    const int steps = min(4, ti.ksteps - kb * 4);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < steps)
                            umma_f16(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                    issued_any = true;
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&accf[abuf]);
                if (++abuf == ACC_BUFS) { abuf = 0; aphase ^= 1u; }
            }
            if (!ok && issued_any) {
                umma_commit(drain);
                volatile int no_abort = 0;
                mbar_wait_bounded(drain, 0, &no_abort, nullptr, kDrainTimeoutNs);
            }
        }
        __syncwarp();
    } else {
        // ================= epilogue (warps 2..9; TMEM lane quadrant = warp % 4)
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r_local = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        int abuf = 0;
        uint32_t aphase = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const Tile ti = decode<TR::krag>(tile, p, seg, nseg);
            const GroupDev& g = p.g[ti.grp];
            const bool row_ok = r_local < ti.rows_ok;
            const int n_valid = g.N - ti.n0;
            if (!warp_wait(&accf[abuf], aphase, abort_flag, p.status, p.timeout_ns, lane)) break;
            tc_fence_after();
            const long long row_off = ti.c_off + static_cast<long long>(r_local) * ti.ldc;
#pragma unroll 1
            for (int cc = 0; cc < 2; ++cc) {
                const int c0 = half * 4 + cc * 2;
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
                    const int c = c0 + u;
                    if (!row_ok || c * 32 >= n_valid) continue;
                    const long long off = row_off + c * 32;
                    if constexpr (MODE == MODE_RECOMP) {
                        const float* bias = g.bias + static_cast<long long>(ti.mat) * g.N + ti.n0 + c * 32;
                        uint32_t ph[16], pd[16];
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 b4 = __ldg(reinterpret_cast<const float4*>(bias) + j4);
                            const float v0 = __uint_as_float(r[u][4 * j4 + 0]) + b4.x;
                            const float v1 = __uint_as_float(r[u][4 * j4 + 1]) + b4.y;
                            const float v2 = __uint_as_float(r[u][4 * j4 + 2]) + b4.z;
                            const float v3 = __uint_as_float(r[u][4 * j4 + 3]) + b4.w;
                            ph[2 * j4] = pack_bf16x2(silu_fast(v0), silu_fast(v1));
                            ph[2 * j4 + 1] = pack_bf16x2(silu_fast(v2), silu_fast(v3));
                            pd[2 * j4] = pack_bf16x2(dsilu_fast(v0), dsilu_fast(v1));
                            pd[2 * j4 + 1] = pack_bf16x2(dsilu_fast(v2), dsilu_fast(v3));
                        }
                        uint4* dh = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out0) + off);
                        uint4* dd = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out1) + off);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            dh[q] = make_uint4(ph[4 * q], ph[4 * q + 1], ph[4 * q + 2], ph[4 * q + 3]);
                            dd[q] = make_uint4(pd[4 * q], pd[4 * q + 1], pd[4 * q + 2], pd[4 * q + 3]);
                        }
                    } else if constexpr (MODE == MODE_DSILU) {
                        const uint4* sp = reinterpret_cast<const uint4*>(g.aux + off);
                        uint32_t po[16];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 s4 = __ldg(sp + q);
                            const uint32_t sw[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                            for (int w = 0; w < 4; ++w) {
                                const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&sw[w]);
                                const float2 sf = __bfloat1622float2(s2);
                                const int j = 8 * q + 2 * w;
                                po[4 * q + w] = pack_bf16x2(__uint_as_float(r[u][j]) * sf.x,
                                                            __uint_as_float(r[u][j + 1]) * sf.y);
                            }
                        }
                        uint4* dz = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out0) + off);
#pragma unroll
                        for (int q = 0; q < 4; ++q) dz[q] = make_uint4(po[4 * q], po[4 * q + 1], po[4 * q + 2], po[4 * q + 3]);
                    } else if (MODE == MODE_DX && g.out_bf16) {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out0) + off);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(
                                pack_bf16x2(__uint_as_float(r[u][8 * q + 0]), __uint_as_float(r[u][8 * q + 1])),
                                pack_bf16x2(__uint_as_float(r[u][8 * q + 2]), __uint_as_float(r[u][8 * q + 3])),
                                pack_bf16x2(__uint_as_float(r[u][8 * q + 4]), __uint_as_float(r[u][8 * q + 5])),
                                pack_bf16x2(__uint_as_float(r[u][8 * q + 6]), __uint_as_float(r[u][8 * q + 7])));
                    } else {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(g.out0) + off);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            dst[q] = make_float4(__uint_as_float(r[u][4 * q]), __uint_as_float(r[u][4 * q + 1]),
                                                 __uint_as_float(r[u][4 * q + 2]), __uint_as_float(r[u][4 * q + 3]));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&acce[abuf]);
            if (++abuf == ACC_BUFS) { abuf = 0; aphase ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem_base);
    }
}

// Host: device copy of a group and its tensor maps.
bool fill_group(Params& p, int gi, const BwdGemmGroup& h, bool a_mn, bool b_mn) {
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
    // 256 rows of N, MN-major boxes of 64 N x 64 rows of K
    if (!encode_tma_2d(&p.a_map[gi], h.A, h.a_rows, h.a_cols, 2, a_mn ? 64 : BM)) return false;
    if (!encode_tma_3d(&p.b_map[gi], h.B, h.b_mats, h.b_rows, h.b_cols, 2, b_mn ? 64 : BN)) return false;
    return true;
}

template <int MODE>
cudaError_t launch_mode(const BwdGemmArgs& a, cudaStream_t st) {
    using TR = ModeTraits<MODE>;
    Params p;
    std::memset(&p, 0, sizeof(p));
    for (int gi = 0; gi < 2; ++gi)
        if (!fill_group(p, gi, a.g[gi], TR::a_mn, TR::b_mn)) return cudaErrorInvalidValue;
    int tiles[2] = {0, 0};
    for (int gi = 0; gi < 2; ++gi) {
        const BwdGemmGroup& g = a.g[gi];
        if (g.n_mats > 0 && TR::krag) tiles[gi] = g.n_mats * ((g.M + BM - 1) / BM) * ((g.N + BN - 1) / BN);
    }
    p.tiles0 = tiles[0];
    p.tiles_total = tiles[0] + tiles[1];
    p.status = a.status;
    p.timeout_ns = kWaitTimeoutNs;
    constexpr int smem = Smem::ALLOC;
    cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(bwd_gemm_kernel<MODE>, dim3(device_sm_count()), dim3(NUM_THREADS), smem, st, 1, p);
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

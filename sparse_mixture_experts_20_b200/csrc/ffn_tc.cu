// Grouped expert FFN GEMMs on the 5th-generation tensor cores (tcgen05).
//
// "論文解説: DeepSeekMoE" §アルゴリズム: each expert is Linear(d, d_ff) + bias
// -> SiLU -> Linear(d_ff, d) + bias.  "DeepSeek DeepEP" §DeepEP とは item 5 /
// §DeepEP の性能: FP8 dispatch, BF16 combine.
//
// One persistent kernel computes C = epilogue(A B^T + bias) over a list of
// ragged row segments: one segment per routed expert (rows taken from the
// device-side dispatch offsets, so the host never synchronises) followed by
// one segment per shared expert (T rows each).  The tile list is
// (segment, n-tile, m-tile) with m fastest, so CTAs running at the same time
// share an expert's weight tile through L2.
//
// Per CTA (192 threads, one CTA per SM):
//   warp 0      TMA producer: A tile (128 rows x 128 bytes) and B tile
//               (BN rows x 128 bytes), 128-byte swizzle, into a ring of
//               shared-memory stages guarded by full/empty mbarriers;
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M=128) into
//               tensor memory and frees each stage with tcgen05.commit;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (thread = row),
//               bias, SiLU, rounding/quantisation and 16-byte stores.
// Rows of a tile past the end of its segment are computed (they belong to
// the next segment or read as zeros) and never stored.
//
// BF16 engine: BN = 256, fp32 accumulation over the whole K loop in one of
// two 256-column TMEM buffers (the epilogue of tile i overlaps the MMAs of
// tile i+1).
// FP8 engine: e4m3 x e4m3 (kind::f8f6f4), BN = 128.  The operand scales
// change every 128 columns of K (activation: per row; weight: per 128x128
// block), so each 128-wide K block is accumulated on its own into one of four
// 128-column TMEM buffers and the epilogue warps fold it into fp32 registers
// with scale_a[row] * scale_b: acc += sa * sb * partial.
//
// Every wait is bounded (see common.cuh); on expiry the CTA drains its
// in-flight copies and MMAs, frees its tensor memory and exits, and the host
// sees MOE_DEV_TIMEOUT in the workspace status word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cstring>
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int NUM_THREADS = 192;
constexpr int MAX_SEGS = 256 + 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;    // 2 s per wait
constexpr uint64_t kDrainTimeoutNs = 200000000ull;    // 0.2 s while unwinding

template <bool FP8> struct Cfg;
template <> struct Cfg<false> {          // bf16
    static constexpr int BN = 256, BK = 64, STAGES = 4, ACC_BUFS = 2;
    static constexpr int ELEM = 2;
};
template <> struct Cfg<true> {           // e4m3
    static constexpr int BN = 128, BK = 128, STAGES = 6, ACC_BUFS = 4;
    static constexpr int ELEM = 1;
};

struct GroupDev {
    int n_mats;
    const int32_t* offsets;   // routed: (n_mats+1); fixed group: nullptr
    int fixed_rows;
    int a_row_base, a_seg_stride;
    const float* a_scales;    // FP8 (a_rows, K/128)
    const float* b_scales;    // FP8 (n_mats, N/128, K/128)
    const float* bias;        // (n_mats, N)
    void* C;
    int c_row_base;
    float* c_scales;          // FP8 first layer (c_rows, N/128)
    int N, K;
};

struct __align__(64) TcParams {
    CUtensorMap a_map[2];
    CUtensorMap b_map[2];
    GroupDev g[2];
    int silu;
    int out_fp8;
    int32_t* status;
    uint64_t timeout_ns;
};

struct TileInfo {
    int grp, mat, rows_left, a_row, c_row, n0, kblocks;
};

template <bool FP8>
struct Smem {
    static constexpr int BN = Cfg<FP8>::BN, STAGES = Cfg<FP8>::STAGES;
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
    // full[STAGES], empty[STAGES], accf[4], acce[4], drain
    static constexpr int N_BARS = 2 * STAGES + 4 + 4 + 1;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;   // tmem addr, abort flag, nseg
    static constexpr int OFF_SEG = OFF_MISC + 16;
    // seg_start[MAX_SEGS+1], seg_rows, seg_arow, seg_crow, seg_mat (MAX_SEGS each)
    static constexpr int SEG_INTS = (MAX_SEGS + 1) + 4 * MAX_SEGS;
    static constexpr int TOTAL = OFF_SEG + SEG_INTS * 4;
    static constexpr int ALLOC = TOTAL + 1024;               // slack for 1 KB alignment
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

template <bool FP8>
__device__ __forceinline__ int ntiles_of(const GroupDev& g) {
    return ceil_div(g.N, Cfg<FP8>::BN);
}

template <bool FP8>
__device__ __forceinline__ TileInfo decode_tile(int tile, const TcParams& p, const int* seg_start,
                                                const int* seg_rows, const int* seg_arow,
                                                const int* seg_crow, const int* seg_mat, int nseg) {
    int lo = 0, hi = nseg - 1;                      // last s with seg_start[s] <= tile
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seg_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int s = lo;
    const int local = tile - seg_start[s];
    const int mtiles = ceil_div(seg_rows[s], BM);
    const int nt = local / mtiles, mt = local % mtiles;
    TileInfo ti;
    ti.grp = seg_mat[s] >> 16;
    ti.mat = seg_mat[s] & 0xFFFF;
    ti.rows_left = seg_rows[s] - mt * BM;
    ti.a_row = seg_arow[s] + mt * BM;
    ti.c_row = seg_crow[s] + mt * BM;
    ti.n0 = nt * Cfg<FP8>::BN;
    ti.kblocks = ceil_div(p.g[ti.grp].K, Cfg<FP8>::BK);
    return ti;
}

// Bounded wait done by lane 0 only; the result is broadcast so that the warp
// leaves converged (the tcgen05.ld that follows is warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, uint64_t timeout_ns, int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(bar, parity, abort_flag, status, timeout_ns) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

template <bool FP8>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_ffn_tc_kernel(const __grid_constant__ TcParams p) {
    using C = Cfg<FP8>;
    using L = Smem<FP8>;
    constexpr int BN = C::BN, STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* accf = bars + 2 * STAGES;
    uint64_t* acce = accf + 4;
    uint64_t* drain = acce + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    int* seg_start = reinterpret_cast<int*>(smem + L::OFF_SEG);
    int* seg_rows = seg_start + MAX_SEGS + 1;
    int* seg_arow = seg_rows + MAX_SEGS;
    int* seg_crow = seg_arow + MAX_SEGS;
    int* seg_mat = seg_crow + MAX_SEGS;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- prologue: TMEM, barriers, segment table
    if (warp == 0) tmem_alloc<TMEM_COLS>(tmem_slot);
    if (warp == 1 && lane == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 4; ++i) { mbar_init(&accf[i], 1); mbar_init(&acce[i], 128); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int gi = 0; gi < 2; ++gi) {
            if (p.g[gi].n_mats > 0) { tma_prefetch_desc(&p.a_map[gi]); tma_prefetch_desc(&p.b_map[gi]); }
        }
    }
    const int n0segs = p.g[0].n_mats, n1segs = p.g[1].n_mats;
    const int nseg = n0segs + n1segs;
    for (int s = tid; s < nseg; s += NUM_THREADS) {
        int rows, arow, crow, packed;
        if (s < n0segs) {
            const GroupDev& g = p.g[0];
            const int o0 = g.offsets[s], o1 = g.offsets[s + 1];
            rows = o1 - o0;
            arow = g.a_row_base + o0;
            crow = g.c_row_base + o0;
            packed = s;
        } else {
            const GroupDev& g = p.g[1];
            const int i = s - n0segs;
            rows = g.fixed_rows;
            arow = g.a_row_base + i * g.a_seg_stride;
            crow = g.c_row_base + i * g.fixed_rows;
            packed = (1 << 16) | i;
        }
        seg_rows[s] = rows;
        seg_arow[s] = arow;
        seg_crow[s] = crow;
        seg_mat[s] = packed;
        const int nt = (s < n0segs) ? ntiles_of<FP8>(p.g[0]) : ntiles_of<FP8>(p.g[1]);
        seg_start[s + 1] = ceil_div(rows, BM) * nt;     // tile count, scanned below
    }
    __syncthreads();
    if (warp == 0) {                                     // inclusive scan of tile counts
        int carry = 0;
        for (int base = 0; base < nseg; base += 32) {
            const int i = base + lane;
            int v = (i < nseg) ? seg_start[i + 1] : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, v, off);
                if (lane >= off) v += o;
            }
            if (i < nseg) seg_start[i + 1] = v + carry;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) seg_start[0] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total_tiles = seg_start[nseg];

    if (warp == 0) {
        // ================= TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile<FP8>(tile, p, seg_start, seg_rows, seg_arow, seg_crow, seg_mat, nseg);
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[stage], L::A_BYTES + L::B_BYTES);
                    tma_load_2d(smem + L::OFF_A + stage * L::A_BYTES, &p.a_map[ti.grp], &full[stage],
                                kb * C::BK, ti.a_row);
                    tma_load_3d(smem + L::OFF_B + stage * L::B_BYTES, &p.b_map[ti.grp], &full[stage],
                                kb * C::BK, ti.n0, ti.mat);
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
            constexpr uint32_t idesc = FP8 ? make_idesc(0, BM, BN) : make_idesc(1, BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int abuf = 0;
            uint32_t aphase = 0;
            bool ok = true, issued_any = false;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile<FP8>(tile, p, seg_start, seg_rows, seg_arow, seg_crow, seg_mat, nseg);
                if (!FP8) {
                    if (!mbar_wait_bounded(&acce[abuf], aphase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    tc_fence_after();
                }
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (FP8) {
                        if (!mbar_wait_bounded(&acce[abuf], aphase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                        tc_fence_after();
                    }
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_k_sw128(smem + L::OFF_A + stage * L::A_BYTES);
                    const uint64_t bdesc = smem_desc_k_sw128(smem + L::OFF_B + stage * L::B_BYTES);
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * BN);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {            // 4 x 32 bytes of K per stage
                        const uint32_t acc = FP8 ? (k > 0) : (kb > 0 || k > 0);
                        if (FP8) umma_f8(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
                        else     umma_f16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
                    }
                    issued_any = true;
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    if (FP8) {
                        umma_commit(&accf[abuf]);
                        if (++abuf == C::ACC_BUFS) { abuf = 0; aphase ^= 1u; }
                    }
                }
                if (!ok) break;
                if (!FP8) {
                    umma_commit(&accf[abuf]);
                    if (++abuf == C::ACC_BUFS) { abuf = 0; aphase ^= 1u; }
                }
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
        // ================= epilogue (warps 2..5; TMEM lane quadrant = warp % 4)
        const int quad = warp & 3;
        const int r_local = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        int abuf = 0;
        uint32_t aphase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            const TileInfo ti = decode_tile<FP8>(tile, p, seg_start, seg_rows, seg_arow, seg_crow, seg_mat, nseg);
            const GroupDev& g = p.g[ti.grp];
            const bool row_ok = r_local < ti.rows_left;
            const int n_valid = min(BN, g.N - ti.n0);
            if (!FP8) {
                if (!warp_wait(&accf[abuf], aphase, abort_flag, p.status, p.timeout_ns, lane)) { ok = false; break; }
                tc_fence_after();
                __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(g.C) +
                                      static_cast<size_t>(ti.c_row + r_local) * g.N + ti.n0;
                const float* bias = g.bias + static_cast<size_t>(ti.mat) * g.N + ti.n0;
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(abuf * BN + c * 32), r);
                    tmem_ld_wait();
                    if (row_ok && c * 32 < n_valid) {
                        uint32_t packed[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            float v0 = __uint_as_float(r[2 * j]) + __ldg(bias + c * 32 + 2 * j);
                            float v1 = __uint_as_float(r[2 * j + 1]) + __ldg(bias + c * 32 + 2 * j + 1);
                            if (p.silu) { v0 = silu_f32(v0); v1 = silu_f32(v1); }
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
                            packed[j] = *reinterpret_cast<uint32_t*>(&h2);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(crow + c * 32);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                    }
                }
                tc_fence_before();
                mbar_arrive(&acce[abuf]);
                if (++abuf == C::ACC_BUFS) { abuf = 0; aphase ^= 1u; }
            } else {
                float acc[BN];
#pragma unroll
                for (int j = 0; j < BN; ++j) acc[j] = 0.f;
                const int kq = g.K / 128;
                const float* sa_row = g.a_scales + static_cast<size_t>(ti.a_row + r_local) * kq;
                const float* sb = g.b_scales + (static_cast<size_t>(ti.mat) * (g.N / 128) + ti.n0 / 128) * kq;
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    const float sa = row_ok ? __ldg(sa_row + kb) : 0.f;
                    const float scale = sa * __ldg(sb + kb);
                    if (!warp_wait(&accf[abuf], aphase, abort_flag, p.status, p.timeout_ns, lane)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(abuf * BN + c * 32), r);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) acc[c * 32 + j] = fmaf(scale, __uint_as_float(r[j]), acc[c * 32 + j]);
                    }
                    tc_fence_before();
                    mbar_arrive(&acce[abuf]);
                    if (++abuf == C::ACC_BUFS) { abuf = 0; aphase ^= 1u; }
                }
                if (!ok) break;
                if (row_ok && n_valid == BN) {
                    const float* bias = g.bias + static_cast<size_t>(ti.mat) * g.N + ti.n0;
                    if (p.out_fp8) {
                        // first layer: bias + SiLU, then one e4m3 block of 128 columns per row
                        float amax = 0.f;
#pragma unroll
                        for (int j = 0; j < BN; ++j) {
                            acc[j] = silu_f32(acc[j] + __ldg(bias + j));
                            amax = fmaxf(amax, fabsf(acc[j]));
                        }
                        const float sc = pow2_scale_448(amax);
                        const float inv = 1.0f / sc;             // exact: sc is a power of two
                        uint8_t* crow = static_cast<uint8_t*>(g.C) +
                                        static_cast<size_t>(ti.c_row + r_local) * g.N + ti.n0;
#pragma unroll
                        for (int q = 0; q < BN / 16; ++q) {
                            uint32_t w[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const int j = q * 16 + h * 4;
                                const uint32_t lo = f32x2_to_e4m3x2(acc[j] * inv, acc[j + 1] * inv);
                                const uint32_t hi = f32x2_to_e4m3x2(acc[j + 2] * inv, acc[j + 3] * inv);
                                w[h] = lo | (hi << 16);
                            }
                            reinterpret_cast<uint4*>(crow)[q] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                        g.c_scales[static_cast<size_t>(ti.c_row + r_local) * (g.N / 128) + ti.n0 / 128] = sc;
                    } else {
                        // second layer: bias, bf16 output
                        __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(g.C) +
                                              static_cast<size_t>(ti.c_row + r_local) * g.N + ti.n0;
#pragma unroll
                        for (int q = 0; q < BN / 8; ++q) {
                            uint32_t w[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const int j = q * 8 + h * 2;
                                __nv_bfloat162 v = __floats2bfloat162_rn(acc[j] + __ldg(bias + j),
                                                                         acc[j + 1] + __ldg(bias + j + 1));
                                w[h] = *reinterpret_cast<uint32_t*>(&v);
                            }
                            reinterpret_cast<uint4*>(crow)[q] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            }
        }
        (void)ok;
    }

    // ---- teardown: every role is done with TMEM
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem_base);
    }
}

// ------------------------------------------------------------------ host side

template <bool FP8>
cudaError_t launch_tc(const GemmArgs& a, cudaStream_t st) {
    using C = Cfg<FP8>;
    TcParams p;
    std::memset(&p, 0, sizeof(p));
    for (int gi = 0; gi < 2; ++gi) {
        const GemmGroup& g = a.g[gi];
        GroupDev& d = p.g[gi];
        d.n_mats = g.n_mats;
        if (g.n_mats == 0) continue;
        d.offsets = g.offsets;
        d.fixed_rows = g.fixed_rows;
        d.a_row_base = g.a_row_base;
        d.a_seg_stride = g.a_seg_stride;
        d.a_scales = g.a_scales;
        d.b_scales = g.b_scales;
        d.bias = g.bias;
        d.C = g.C;
        d.c_row_base = g.c_row_base;
        d.c_scales = g.c_scales;
        d.N = g.N;
        d.K = g.K;
        if (!encode_tma_2d(&p.a_map[gi], g.A, g.a_rows, g.K, C::ELEM, BM)) return cudaErrorInvalidValue;
        if (!encode_tma_3d(&p.b_map[gi], g.B, g.n_mats, g.N, g.K, C::ELEM, C::BN)) return cudaErrorInvalidValue;
    }
    p.silu = a.silu;
    p.out_fp8 = a.out_fp8;
    p.status = a.status;
    p.timeout_ns = kWaitTimeoutNs;
    constexpr int smem = Smem<FP8>::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(grouped_ffn_tc_kernel<FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    grouped_ffn_tc_kernel<FP8><<<device_sm_count(), NUM_THREADS, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grouped_ffn_bf16(const Dims&, const GemmArgs& a, cudaStream_t st) {
    return launch_tc<false>(a, st);
}

cudaError_t launch_grouped_ffn_fp8(const Dims&, const GemmArgs& a, cudaStream_t st) {
    return launch_tc<true>(a, st);
}

}  // namespace moe

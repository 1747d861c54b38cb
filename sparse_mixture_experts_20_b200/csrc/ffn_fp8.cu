// Grouped expert FFN GEMMs in FP8 e4m3 with block scales, on tcgen05.
//
// "論文解説: DeepSeekMoE" §アルゴリズム: each expert is Linear(d, d_ff) + bias
// -> SiLU -> Linear(d_ff, d) + bias.  "DeepSeek DeepEP" §DeepEP とは item 5
// and §DeepEP の性能: FP8 dispatch, BF16 combine.
//
// Operands: activations e4m3 with one power-of-two scale per row per 128
// columns of K; weights e4m3 with one power-of-two scale per 128x128 block.
// Powers of two are exactly UE8M0, so the scales go to the tensor core
// itself: tcgen05.mma kind::mxf8f6f4.block_scale reads one UE8M0 scale per
// row (of A) and per column (of B) per 32 elements of K from tensor memory,
// and the accumulator sums sa * sb * (a . b) over the whole K loop in fp32.
//
// Per CTA (320 threads, one CTA per SM), tiles of 128 rows x 128 weight rows:
//   warp 0      TMA producer: A and B tiles of 128 rows x 128 bytes (one
//               scale block of K) into a ring of 6 stages;
//   warp 1      MMA issuer: per stage 4 x tcgen05.mma (K = 32 each) with the
//               scale factors of that stage, accumulating in one of two
//               128-column TMEM buffers;
//   warps 2..5  epilogue: tcgen05.ld (thread = row), bias, SiLU and the
//               per-row e4m3 re-quantisation of the hidden activation (one
//               128-column scale block per row and tile, so the amax is
//               thread-local), or bias and bf16 output;
//   warps 6..9  scale-factor writers: per stage, load the 128 row scales of
//               A and the block scale of B (prefetched 8 stages ahead),
//               convert to UE8M0 and tcgen05.st them into a ring of 8
//               tensor-memory slots.  Each slot holds, in every lane quadrant,
//               lane m: columns c = 0..3 = the scale of row 32c + m (A) and of
//               weight row 32c + m (B), each byte repeated for the four
//               32-element sub-blocks of K.
// Every wait is bounded (common.cuh).
#include "ffn_common.cuh"

namespace moe {
namespace {

using namespace ffn;

constexpr int NUM_THREADS = 320;
constexpr int BN = 128, BK = 128, STAGES = 6, ACC_BUFS = 2, SF_SLOTS = 8, LOOKAHEAD = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = ACC_BUFS * BN;          // scale-factor slots after the accumulators
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
constexpr uint64_t kDrainTimeoutNs = 200000000ull;

struct Smem {
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
    // full, empty [STAGES]; accf, acce [ACC_BUFS]; sff, sfe [SF_SLOTS]; drain
    static constexpr int N_BARS = 2 * STAGES + 2 * ACC_BUFS + 2 * SF_SLOTS + 1;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int OFF_SEG = OFF_MISC + 16;
    static constexpr int TOTAL = OFF_SEG + SegTable::SEG_INTS * 4;
    static constexpr int ALLOC = TOTAL + 1024;
};

// A positive power-of-two fp32 scale as a UE8M0 byte (its biased exponent),
// repeated in the four bytes of a 32-bit word.
__device__ __forceinline__ uint32_t ue8m0_x4(float s) {
    return ((__float_as_uint(s) >> 23) & 0xFFu) * 0x01010101u;
}

struct ItemIt {
    int tile, kb;
    TileInfo ti;
};

__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_ffn_fp8_kernel(const __grid_constant__ TcParams p) {
    using L = Smem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = full + STAGES;
    uint64_t* accf = empty + STAGES;
    uint64_t* acce = accf + ACC_BUFS;
    uint64_t* sff = acce + ACC_BUFS;
    uint64_t* sfe = sff + SF_SLOTS;
    uint64_t* drain = sfe + SF_SLOTS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    SegTable seg(reinterpret_cast<int*>(smem + L::OFF_SEG));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 0) tmem_alloc<TMEM_COLS>(tmem_slot);
    if (warp == 1 && lane == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < ACC_BUFS; ++i) { mbar_init(&accf[i], 1); mbar_init(&acce[i], 128); }
        for (int i = 0; i < SF_SLOTS; ++i) { mbar_init(&sff[i], 128); mbar_init(&sfe[i], 1); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int gi = 0; gi < 2; ++gi)
            if (p.g[gi].n_mats > 0) { tma_prefetch_desc(&p.a_map[gi]); tma_prefetch_desc(&p.b_map[gi]); }
    }
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
            constexpr uint32_t idesc = make_idesc_mxf8(BM, BN);
            int stage = 0, abuf = 0, sslot = 0;
            uint32_t phase = 0, aphase = 0, sphase = 0;
            bool ok = true, issued_any = false;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile<BN, BK>(tile, p, seg, nseg);
                if (!mbar_wait_bounded(&acce[abuf], aphase ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * BN);
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    if (!mbar_wait_bounded(&sff[sslot], sphase, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_k_sw128(smem + L::OFF_A + stage * L::A_BYTES);
                    const uint64_t bdesc = smem_desc_k_sw128(smem + L::OFF_B + stage * L::B_BYTES);
                    const uint32_t sfa = tmem_base + SF_COL0 + static_cast<uint32_t>(sslot * 8);
#pragma unroll
                    for (int k = 0; k < 4; ++k)            // 4 x 32 e4m3 of K per stage
                        umma_mxf8_bs(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, sfa, sfa + 4,
                                     (kb > 0 || k > 0) ? 1u : 0u);
                    issued_any = true;
                    umma_commit(&empty[stage]);
                    umma_commit(&sfe[sslot]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    if (++sslot == SF_SLOTS) { sslot = 0; sphase ^= 1u; }
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
    } else if (warp < 6) {
        // ================= epilogue (warps 2..5)
        const int quad = warp & 3;
        const int r_local = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        int abuf = 0;
        uint32_t aphase = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const TileInfo ti = decode_tile<BN, BK>(tile, p, seg, nseg);
            const GroupDev& g = p.g[ti.grp];
            const bool row_ok = r_local < ti.rows_left;
            if (!warp_wait(&accf[abuf], aphase, abort_flag, p.status, p.timeout_ns, lane)) break;
            tc_fence_after();
            const float* bias = g.bias + static_cast<size_t>(ti.mat) * g.N + ti.n0;
            const uint32_t acc_col = static_cast<uint32_t>(abuf * BN);
            if (p.out_fp8) {
                // first layer: bias + SiLU, then one e4m3 block of 128 columns per row
                float v[BN];
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(lane_base + acc_col + static_cast<uint32_t>(c * 32), r);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[c * 32 + j] = __uint_as_float(r[j]);
                }
                tc_fence_before();
                mbar_arrive(&acce[abuf]);                    // accumulator copied out
                if (row_ok) {
                    float amax = 0.f;
#pragma unroll
                    for (int j = 0; j < BN; ++j) {
                        v[j] = silu_f32(v[j] + __ldg(bias + j));
                        amax = fmaxf(amax, fabsf(v[j]));
                    }
                    const float sc = pow2_scale_448(amax);
                    const float inv = 1.0f / sc;             // exact: sc is a power of two
                    uint8_t* crow = static_cast<uint8_t*>(g.C) + static_cast<size_t>(ti.c_row + r_local) * g.N + ti.n0;
#pragma unroll
                    for (int q = 0; q < BN / 16; ++q) {
                        uint32_t w[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const int j = q * 16 + h * 4;
                            const uint32_t lo = f32x2_to_e4m3x2(v[j] * inv, v[j + 1] * inv);
                            const uint32_t hi = f32x2_to_e4m3x2(v[j + 2] * inv, v[j + 3] * inv);
                            w[h] = lo | (hi << 16);
                        }
                        reinterpret_cast<uint4*>(crow)[q] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                    g.c_scales[static_cast<size_t>(ti.c_row + r_local) * (g.N / 128) + ti.n0 / 128] = sc;
                }
            } else {
                // second layer: bias, bf16 output
                __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(g.C) +
                                      static_cast<size_t>(ti.c_row + r_local) * g.N + ti.n0;
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(lane_base + acc_col + static_cast<uint32_t>(c * 32), r);
                    tmem_ld_wait();
                    if (row_ok) {
                        uint32_t packed[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(
                                __uint_as_float(r[2 * j]) + __ldg(bias + c * 32 + 2 * j),
                                __uint_as_float(r[2 * j + 1]) + __ldg(bias + c * 32 + 2 * j + 1));
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
            }
            if (++abuf == ACC_BUFS) { abuf = 0; aphase ^= 1u; }
        }
    } else {
        // ================= scale-factor writers (warps 6..9)
        const int quad = warp & 3;
        const uint32_t sf_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + SF_COL0;
        auto valid = [&](const ItemIt& it) { return it.tile < total_tiles; };
        auto start = [&](ItemIt& it) {
            it.tile = blockIdx.x;
            it.kb = 0;
            if (it.tile < total_tiles) it.ti = decode_tile<BN, BK>(it.tile, p, seg, nseg);
        };
        auto advance = [&](ItemIt& it) {
            if (++it.kb >= it.ti.kblocks) {
                it.kb = 0;
                it.tile += gridDim.x;
                if (it.tile < total_tiles) it.ti = decode_tile<BN, BK>(it.tile, p, seg, nseg);
            }
        };
        auto load = [&](const ItemIt& it, float (&a)[4], float& b) {
            const GroupDev& g = p.g[it.ti.grp];
            const int kq = g.K / 128;
            const int rows_valid = min(BM, it.ti.rows_left);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int r = 32 * c + lane;
                a[c] = (r < rows_valid) ? __ldg(g.a_scales + static_cast<size_t>(it.ti.a_row + r) * kq + it.kb) : 1.0f;
            }
            b = __ldg(g.b_scales + (static_cast<size_t>(it.ti.mat) * (g.N / 128) + it.ti.n0 / 128) * kq + it.kb);
        };
        ItemIt cur, ahead;
        start(cur);
        start(ahead);
        float ra[LOOKAHEAD][4], rb[LOOKAHEAD];
#pragma unroll
        for (int j = 0; j < LOOKAHEAD; ++j) {
            if (valid(ahead)) { load(ahead, ra[j], rb[j]); advance(ahead); }
        }
        int sslot = 0;
        uint32_t sphase = 0;
        bool ok = true;
        while (ok && valid(cur)) {
#pragma unroll
            for (int j = 0; j < LOOKAHEAD; ++j) {
                if (!valid(cur)) break;
                const uint32_t wa0 = ue8m0_x4(ra[j][0]), wa1 = ue8m0_x4(ra[j][1]);
                const uint32_t wa2 = ue8m0_x4(ra[j][2]), wa3 = ue8m0_x4(ra[j][3]);
                const uint32_t wb = ue8m0_x4(rb[j]);
                if (valid(ahead)) { load(ahead, ra[j], rb[j]); advance(ahead); }
                if (!warp_wait(&sfe[sslot], sphase ^ 1u, abort_flag, p.status, p.timeout_ns, lane)) { ok = false; break; }
                tc_fence_after();
                tmem_st_32x32b_x4(sf_base + static_cast<uint32_t>(sslot * 8), wa0, wa1, wa2, wa3);
                tmem_st_32x32b_x4(sf_base + static_cast<uint32_t>(sslot * 8 + 4), wb, wb, wb, wb);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&sff[sslot]);
                if (++sslot == SF_SLOTS) { sslot = 0; sphase ^= 1u; }
                advance(cur);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem_base);
    }
}

}  // namespace

cudaError_t launch_grouped_ffn_fp8(const Dims&, const GemmArgs& a, cudaStream_t st) {
    TcParams p;
    if (!fill_params(p, a, 1, BN, kWaitTimeoutNs)) return cudaErrorInvalidValue;
    constexpr int smem = Smem::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(grouped_ffn_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    grouped_ffn_fp8_kernel<<<device_sm_count(), NUM_THREADS, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace moe

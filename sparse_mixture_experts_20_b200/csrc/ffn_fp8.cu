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
// Tiles are 128 rows x 256 weight rows: one MMA instruction (K = 32) is then
// about 128 tensor-core cycles of work, enough to hide the cost of issuing
// it from a single thread.  Two 256-column accumulators and the scale-factor
// slots do not fit in the 512 columns of tensor memory, so the accumulators
// overlap: buffer 0 is columns 0..255, buffer 1 columns 192..447, scale slots
// 448..511.  The epilogue drains a tile's 64 overlapping columns first and
// says so on the `ovl` barrier; the MMA of the next tile (in the other
// buffer) starts then, while the epilogue finishes the rest.
//
// Per CTA (320 threads, one CTA per SM):
//   warp 0      TMA producer: A (128 rows x 128 bytes, one scale block of K)
//               and B (256 rows x 128 bytes) into a ring of 4 stages;
//   warp 1      MMA issuer: per stage 4 x tcgen05.mma (K = 32 each) with the
//               scale factors of that stage;
//   warps 2..5  epilogue: tcgen05.ld (thread = row; the overlapping columns
//               first), bias, SiLU and the
//               per-row e4m3 re-quantisation of the hidden activation (one
//               scale per row per 128 columns, so the amax is thread-local),
//               or bias and bf16 output;
//   warps 6..9  scale-factor writers: per stage, the 128 row scales of A and
//               the two block scales of B (prefetched 4 stages ahead: where
//               K is a multiple of 512, as one float4 per row covering four
//               k-blocks, else per stage in a register ring that the loop,
//               unrolled over one turn, reloads slot by slot in place) as
//               UE8M0, written with tcgen05.st into the stage's slot of
//               tensor memory; they arrive on the stage's full barrier next to
//               the TMA bytes, and wait on its empty barrier like the
//               producer.  Slot layout, in every lane quadrant, lane m:
//               columns c = 0..3 hold the scale of A row 32c + m, columns
//               4 + c and 8 + c the scale of weight row 32c + m and
//               128 + 32c + m, each byte repeated for the four 32-element
//               sub-blocks of K.
// Every wait is bounded (common.cuh).
#include "ffn_common.cuh"

namespace moe {
namespace {

using namespace ffn;

constexpr int NUM_THREADS = 320;
constexpr int BK = 128, STAGES = 4, LOOKAHEAD = 4;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_STRIDE = 16;                   // columns per stage slot (4 A + 8 B, padded)
constexpr uint32_t FULL_ARRIVALS = 1 + 4;            // TMA expect_tx + one lane per scale-factor warp
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
constexpr uint64_t kDrainTimeoutNs = 200000000ull;

// Tile geometry by the width BN of the weight tile: 256 (two accumulators
// overlapping by 64 tensor-memory columns, see above) or 128 (two disjoint
// accumulators, for batches with few rows per expert, where the number of
// tiles -- not the work per tile -- decides how evenly the SMs are loaded).
template <int BN_> struct FCfg {
    static constexpr int BN = BN_;
    static constexpr bool OVERLAP = BN == 256;
    static constexpr uint32_t ACC1_COL = OVERLAP ? 192u : static_cast<uint32_t>(BN);   // buffer 1
    static constexpr uint32_t SF_COL0 = ACC1_COL + BN;   // scale-factor slots after the accumulators
    static_assert(BN == 128 || BN == 256, "weight tile width");
    static_assert(SF_COL0 + STAGES * SF_STRIDE <= TMEM_COLS, "tensor memory budget");
    static_assert(!OVERLAP || BN - ACC1_COL == 64, "the epilogue drains two 32-column chunks first");
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
    // full, empty [STAGES]; accf, acce [2]; ovl; drain
    static constexpr int N_BARS = 2 * STAGES + 4 + 2;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int OFF_SEG = OFF_MISC + 16;
    // per epilogue warp, 2 x BN fp32: the biases of its two tiles in flight
    // (read and written as float4: 16-byte aligned)
    static constexpr int OFF_BIAS = (OFF_SEG + SegTable::SEG_INTS * 4 + 15) & ~15;
    // per epilogue warp, two 2 KB staging buffers (32 rows x 64 bytes, 64-byte
    // swizzled) for the TMA stores of its output rows
    static constexpr int OFF_STAGE = (OFF_BIAS + 4 * 2 * BN * 4 + 1023) & ~1023;
    static constexpr int STAGE_BUF = 32 * 64;
    static constexpr int TOTAL = OFF_STAGE + 4 * 2 * STAGE_BUF;
    static constexpr int ALLOC = TOTAL + 1024;
    static_assert(OFF_BIAS % 16 == 0 && (BN * 4) % 16 == 0, "float4 access to the bias buffers");
    static_assert(OFF_A % 1024 == 0 && OFF_B % 1024 == 0 && A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0,
                  "128-byte-swizzled TMA tiles start on 1024-byte boundaries");
    static_assert(OFF_BAR % 8 == 0, "mbarriers are 8-byte aligned");
    static_assert(OFF_STAGE % 1024 == 0, "64-byte-swizzled TMA boxes start on 512-byte boundaries");
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

// The MMA thread's wait for a full stage, bounded like mbar_wait_bounded but
// polling without the suspend hint: this thread is on the critical path, and
// the hinted poll (which the waiting roles keep) measured 0.5-0.8 % slower
// for the whole layer on the V3 prefill and decode batches.
static __device__ __noinline__ bool mma_wait_spin(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  int32_t* status, uint64_t timeout_ns) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > timeout_ns) {
                *abort_flag = 1;
                set_device_status(status, MOE_DEV_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool mma_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status,
                                         uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    return mma_wait_spin(bar, parity, abort_flag, status, timeout_ns);
}

// OUT_FP8: the first layer (bias, SiLU, e4m3 re-quantisation of h) or the
// second (bias, bf16 y); one instance each, so that neither carries the
// other's registers and code.
template <int BN, bool OUT_FP8>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_ffn_fp8_kernel(const __grid_constant__ TcParams p) {
    using L = FCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = full + STAGES;
    uint64_t* accf = empty + STAGES;
    uint64_t* acce = accf + 2;
    uint64_t* ovl = acce + 2;
    uint64_t* drain = ovl + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    SegTable seg(reinterpret_cast<int*>(smem + L::OFF_SEG));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 0) tmem_alloc<TMEM_COLS>(tmem_slot);
    if (warp == 1 && lane == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], FULL_ARRIVALS); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&accf[i], 1); mbar_init(&acce[i], 128); }
        mbar_init(ovl, 128);
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
            int stage = 0, abuf = 0;
            uint32_t phase = 0, aph0 = 0, aph1 = 0, ovl_ph = 0;
            bool ok = true, issued_any = false, first = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile<BN, BK>(tile, p, seg, nseg);
                // the previous tile's overlapping columns drained ...
                if (L::OVERLAP && !first) {
                    if (!mbar_wait_bounded(ovl, ovl_ph, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    ovl_ph ^= 1u;
                }
                first = false;
                // ... and this buffer's tile from two tiles back fully drained
                uint32_t& aph = abuf ? aph1 : aph0;
                if (!mbar_wait_bounded(&acce[abuf], aph ^ 1u, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (abuf ? L::ACC1_COL : 0u);
                for (int kb = 0; kb < ti.kblocks; ++kb) {
                    if (!mma_wait(&full[stage], phase, abort_flag, p.status, p.timeout_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_k_sw128(smem + L::OFF_A + stage * L::A_BYTES);
                    const uint64_t bdesc = smem_desc_k_sw128(smem + L::OFF_B + stage * L::B_BYTES);
                    const uint32_t sfa = tmem_base + L::SF_COL0 + static_cast<uint32_t>(stage) * SF_STRIDE;
#pragma unroll
                    for (int k = 0; k < 4; ++k)            // 4 x 32 e4m3 of K per stage
                        umma_mxf8_bs(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, sfa, sfa + 4,
                                     (kb > 0 || k > 0) ? 1u : 0u);
                    issued_any = true;
                    umma_commit(&empty[stage]);             // frees the smem stage and its scale slot
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&accf[abuf]);
                aph ^= 1u;
                abuf ^= 1;
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
        uint32_t fph0 = 0, fph1 = 0;
        // Output rows leave through shared memory and TMA stores: the warp
        // writes its 32 rows x 64 bytes into one of its two staging buffers
        // (16-byte chunk q of row r at chunk q ^ ((r >> 1) & 3): the 64-byte
        // swizzle, which also spreads the writes over the banks) and one lane
        // stores the box.  A buffer is rewritten only after the store issued
        // from it two boxes earlier has read it.
        uint8_t* stg = smem + L::OFF_STAGE + quad * 2 * L::STAGE_BUF;
        int sbuf = 0;
        // the warp's next staging buffer, free to write; this lane's row in it
        auto stage_begin = [&]() -> uint8_t* {
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
            return stg + sbuf * L::STAGE_BUF + lane * 64;
        };
        auto stage_put = [&](uint8_t* row, int q, const uint4& v) {
            *reinterpret_cast<uint4*>(row + ((q ^ ((lane >> 1) & 3)) << 4)) = v;
        };
        auto stage_end = [&](const void* map, int x, int y) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(map, stg + sbuf * L::STAGE_BUF, x, y);
                bulk_commit();
            }
            sbuf ^= 1;
        };
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const TileInfo ti = decode_tile<BN, BK>(tile, p, seg, nseg);
            const GroupDev& g = p.g[ti.grp];
            const bool row_ok = r_local < ti.rows_left;
            // all 32 rows of this warp lie in the segment: TMA stores; else the
            // valid rows are stored one by one (a box would reach into the
            // next segment's rows)
            const bool full_warp = ti.rows_left >= quad * 32 + 32;
            // the tile's BN biases into this warp's shared-memory buffer while the
            // tile's MMAs run (each warp keeps its own copy, so only the warp
            // itself synchronises); the buffer of tile i is rewritten for tile
            // i + 2, after this warp is done with tile i
            float* bias_s = reinterpret_cast<float*>(smem + L::OFF_BIAS) + (quad * 2 + abuf) * BN;
#pragma unroll
            for (int i = 4 * lane; i < BN; i += 128) {
                const float4 v = (ti.n0 + i < g.N)
                    ? __ldg(reinterpret_cast<const float4*>(g.bias + static_cast<size_t>(ti.mat) * g.N + ti.n0 + i))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4*>(bias_s + i) = v;
            }
            __syncwarp();
            uint32_t& fph = abuf ? fph1 : fph0;
            if (!warp_wait(&accf[abuf], fph, abort_flag, p.status, p.timeout_ns, lane)) break;
            fph ^= 1u;
            tc_fence_after();
            // this tile's accumulator; its overlapping columns are 192..255 of
            // buffer 0 (the second half) or 0..63 of buffer 1 (the first half)
            const uint32_t acc = lane_base + (abuf ? L::ACC1_COL : 0u);
            if constexpr (OUT_FP8) {
                // first layer: bias + SiLU, then one e4m3 block per 128 columns
                // per row; the half holding the overlap goes first
#pragma unroll 1
                for (int hi = 0; hi < BN / 128; ++hi) {
                    const int h = (abuf || !L::OVERLAP) ? hi : (BN / 128 - 1 - hi);
                    float v[128];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(acc + static_cast<uint32_t>(h * 128 + c * 32), r);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[c * 32 + j] = __uint_as_float(r[j]);
                    }
                    tc_fence_before();
                    if (L::OVERLAP && hi == 0) mbar_arrive(ovl);  // overlap read: the next tile may start
                    else if (hi == BN / 128 - 1) mbar_arrive(&acce[abuf]);   // fully read: release it
                    const int n_blk = ti.n0 + h * 128;
                    if (!row_ok || n_blk >= g.N) continue;
                    float amax = 0.f;
                    const float4* b4 = reinterpret_cast<const float4*>(bias_s + h * 128);
#pragma unroll
                    for (int j4 = 0; j4 < 32; ++j4) {
                        const float4 b = b4[j4];
                        v[4 * j4 + 0] = silu_fast(v[4 * j4 + 0] + b.x);
                        v[4 * j4 + 1] = silu_fast(v[4 * j4 + 1] + b.y);
                        v[4 * j4 + 2] = silu_fast(v[4 * j4 + 2] + b.z);
                        v[4 * j4 + 3] = silu_fast(v[4 * j4 + 3] + b.w);
                        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[4 * j4]), fabsf(v[4 * j4 + 1])),
                                                 fmaxf(fabsf(v[4 * j4 + 2]), fabsf(v[4 * j4 + 3]))));
                    }
                    const float sc = pow2_scale_448(amax);
                    const float inv = inv_pow2(sc);          // exact: sc is a power of two
                    uint8_t* crow = static_cast<uint8_t*>(g.C) + static_cast<size_t>(ti.c_row + r_local) * g.N + n_blk;
#pragma unroll
                    for (int sub = 0; sub < 2; ++sub) {            // 64 columns (64 bytes) at a time
                        uint8_t* srow = full_warp ? stage_begin() : nullptr;
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const int q = sub * 4 + q4;
                            uint32_t w[4];
#pragma unroll
                            for (int hh = 0; hh < 4; ++hh) {
                                const int j = q * 16 + hh * 4;
                                const uint32_t lo = f32x2_to_e4m3x2(v[j] * inv, v[j + 1] * inv);
                                const uint32_t hi = f32x2_to_e4m3x2(v[j + 2] * inv, v[j + 3] * inv);
                                w[hh] = lo | (hi << 16);
                            }
                            const uint4 val = make_uint4(w[0], w[1], w[2], w[3]);
                            if (full_warp) stage_put(srow, q4, val);
                            else reinterpret_cast<uint4*>(crow)[q] = val;
                        }
                        if (full_warp) stage_end(&p.c_map[ti.grp], n_blk + 64 * sub, ti.c_row + quad * 32);
                    }
                    g.c_scales[static_cast<size_t>(ti.c_row + r_local) * (g.N / 128) + n_blk / 128] = sc;
                }
            } else {
                // second layer: bias, bf16 output.  Chunks of 32 columns, the
                // overlapping ones first; the tensor-memory load of the next
                // chunk is in flight while a chunk is converted and stored.
                __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(g.C) +
                                      static_cast<size_t>(ti.c_row + r_local) * g.N + ti.n0;
                const int n_valid = min(BN, g.N - ti.n0);
                constexpr int NCH = BN / 32;
                auto col_of = [&](int ci) { return (abuf || !L::OVERLAP) ? ci : (ci + 6) & 7; };
                auto store_chunk = [&](const uint32_t (&r)[32], int c) {
                    if (c * 32 >= n_valid || !(full_warp || row_ok)) return;
                    uint32_t packed[16];
                    const float4* b4 = reinterpret_cast<const float4*>(bias_s + c * 32);
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4) {
                        const float4 b = b4[j4];
                        __nv_bfloat162 lo = __floats2bfloat162_rn(__uint_as_float(r[4 * j4 + 0]) + b.x,
                                                                  __uint_as_float(r[4 * j4 + 1]) + b.y);
                        __nv_bfloat162 hi = __floats2bfloat162_rn(__uint_as_float(r[4 * j4 + 2]) + b.z,
                                                                  __uint_as_float(r[4 * j4 + 3]) + b.w);
                        packed[2 * j4] = *reinterpret_cast<uint32_t*>(&lo);
                        packed[2 * j4 + 1] = *reinterpret_cast<uint32_t*>(&hi);
                    }
                    if (full_warp) {
                        uint8_t* srow = stage_begin();
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            stage_put(srow, q, make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2],
                                                          packed[4 * q + 3]));
                        stage_end(&p.c_map[ti.grp], ti.n0 + c * 32, ti.c_row + quad * 32);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(crow + c * 32);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                    }
                };
                // once chunk `loaded` is in registers: after the two overlapping
                // chunks the next tile may start, after the last the
                // accumulator is free
                auto loaded = [&](int ci) {
                    if (L::OVERLAP && ci == 1) {
                        tc_fence_before();
                        mbar_arrive(ovl);
                    } else if (ci == NCH - 1) {
                        tc_fence_before();
                        mbar_arrive(&acce[abuf]);
                    }
                };
                uint32_t r0[32], r1[32];
                tmem_ld_32x32b_x32(acc + static_cast<uint32_t>(col_of(0) * 32), r0);
                tmem_ld_wait_regs(r0);
                loaded(0);
#pragma unroll 1
                for (int ci = 0; ci < NCH; ci += 2) {
                    tmem_ld_32x32b_x32(acc + static_cast<uint32_t>(col_of(ci + 1) * 32), r1);
                    store_chunk(r0, col_of(ci));
                    tmem_ld_wait_regs(r1);
                    loaded(ci + 1);
                    if (ci + 2 < NCH) tmem_ld_32x32b_x32(acc + static_cast<uint32_t>(col_of(ci + 2) * 32), r0);
                    store_chunk(r1, col_of(ci + 1));
                    if (ci + 2 < NCH) {
                        tmem_ld_wait_regs(r0);
                        loaded(ci + 2);
                    }
                }
            }
            abuf ^= 1;
        }
        // the stores have read their buffers and landed before the CTA exits
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    } else {
        // ================= scale-factor writers (warps 6..9)
        const int quad = warp & 3;
        const uint32_t sf_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + L::SF_COL0;
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
        // A: the scales of rows 32c + lane; B: the two weight blocks of the tile
        auto load = [&](const ItemIt& it, float (&a)[4], float (&b)[2]) {
            const GroupDev& g = p.g[it.ti.grp];
            const int kq = g.K / 128;
            const int rows_valid = min(BM, it.ti.rows_left);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int r = 32 * c + lane;
                a[c] = (r < rows_valid) ? __ldg(g.a_scales + static_cast<size_t>(it.ti.a_row + r) * kq + it.kb) : 1.0f;
            }
            const int nb = g.N / 128;
#pragma unroll
            for (int h = 0; h < BN / 128; ++h) {
                const int blk = it.ti.n0 / 128 + h;
                b[h] = (blk < nb) ? __ldg(g.b_scales + (static_cast<size_t>(it.ti.mat) * nb + blk) * kq + it.kb) : 1.0f;
            }
        };
        ItemIt cur, ahead;
        start(cur);
        start(ahead);
        uint32_t phase = 0;
        bool aborted = false;
        if (p.sf_vec) {
            // Every K a multiple of 4 * BK and the scale arrays 16-byte
            // aligned: a row's (or weight block's) scales of four consecutive
            // k-blocks are one float4, so a group of four items takes 6
            // vector loads instead of 24 scalar ones (a quarter of the L1
            // requests: the A loads of a warp touch 32 rows each).  A tile is
            // whole groups, and a group is one turn of the stages.  One group
            // in flight (loaded a group ahead) measured faster than two: the
            // first layer is at the register cap of 10 warps, and the second
            // ring adds spills.
            static_assert(STAGES == 4, "a group of four k-blocks is one turn of the stages");
            constexpr int GROUPS = 1;
            auto advance4 = [&](ItemIt& it) {
                it.kb += 4;
                if (it.kb >= it.ti.kblocks) {
                    it.kb = 0;
                    it.tile += gridDim.x;
                    if (it.tile < total_tiles) it.ti = decode_tile<BN, BK>(it.tile, p, seg, nseg);
                }
            };
            auto load4 = [&](const ItemIt& it, float4 (&a)[4], float4 (&b)[2]) {
                const GroupDev& g = p.g[it.ti.grp];
                const int kq = g.K / 128;
                const int rows_valid = min(BM, it.ti.rows_left);
                const float4 one = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int r = 32 * c + lane;
                    a[c] = (r < rows_valid)
                        ? __ldg(reinterpret_cast<const float4*>(g.a_scales + static_cast<size_t>(it.ti.a_row + r) * kq + it.kb))
                        : one;
                }
                const int nb = g.N / 128;
#pragma unroll
                for (int h = 0; h < BN / 128; ++h) {
                    const int blk = it.ti.n0 / 128 + h;
                    b[h] = (blk < nb)
                        ? __ldg(reinterpret_cast<const float4*>(g.b_scales + (static_cast<size_t>(it.ti.mat) * nb + blk) * kq + it.kb))
                        : one;
                }
            };
            auto comp = [](const float4& v, int q) { return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w; };
            float4 ga[GROUPS][4], gb[GROUPS][2];
#pragma unroll
            for (int j = 0; j < GROUPS; ++j) {
                gb[j][1] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (valid(ahead)) { load4(ahead, ga[j], gb[j]); advance4(ahead); }
            }
#pragma unroll 1
            while (valid(cur) && !aborted) {
#pragma unroll
                for (int j = 0; j < GROUPS; ++j) {
                    if (!valid(cur) || aborted) break;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t wa0 = ue8m0_x4(comp(ga[j][0], q)), wa1 = ue8m0_x4(comp(ga[j][1], q));
                        const uint32_t wa2 = ue8m0_x4(comp(ga[j][2], q)), wa3 = ue8m0_x4(comp(ga[j][3], q));
                        const uint32_t wb0 = ue8m0_x4(comp(gb[j][0], q)), wb1 = ue8m0_x4(comp(gb[j][1], q));
                        if (q == 3 && valid(ahead)) { load4(ahead, ga[j], gb[j]); advance4(ahead); }
                        if (!warp_wait(&empty[q], phase ^ 1u, abort_flag, p.status, p.timeout_ns, lane)) {
                            aborted = true;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t slot = sf_base + static_cast<uint32_t>(q) * SF_STRIDE;
                        tmem_st_32x32b_x4(slot, wa0, wa1, wa2, wa3);
                        tmem_st_32x32b_x4(slot + 4, wb0, wb0, wb0, wb0);
                        if (BN == 256) tmem_st_32x32b_x4(slot + 8, wb1, wb1, wb1, wb1);
                        tmem_st_wait();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&full[q]);
                    }
                    phase ^= 1u;
                    advance4(cur);
                }
            }
        } else {
            float ra[LOOKAHEAD][4], rb[LOOKAHEAD][2] = {};
#pragma unroll
            for (int j = 0; j < LOOKAHEAD; ++j) {
                if (valid(ahead)) { load(ahead, ra[j], rb[j]); advance(ahead); }
            }
            // Item i of the stream uses ring slot i % LOOKAHEAD and stage
            // i % STAGES; LOOKAHEAD is a multiple of STAGES and the loop is
            // unrolled over one turn of the ring, so both indices are constants:
            // a slot's scales (loaded LOOKAHEAD items earlier) are converted and
            // the slot reloaded in place, with no register moves that would wait
            // on a load still in flight.
            static_assert(LOOKAHEAD % STAGES == 0, "a turn of the ring is whole turns of the stages");
#pragma unroll 1
            while (valid(cur) && !aborted) {
#pragma unroll
                for (int j = 0; j < LOOKAHEAD; ++j) {
                    const int stage = j % STAGES;
                    if (!valid(cur)) break;
                    const uint32_t wa0 = ue8m0_x4(ra[j][0]), wa1 = ue8m0_x4(ra[j][1]);
                    const uint32_t wa2 = ue8m0_x4(ra[j][2]), wa3 = ue8m0_x4(ra[j][3]);
                    const uint32_t wb0 = ue8m0_x4(rb[j][0]), wb1 = ue8m0_x4(rb[j][1]);
                    if (valid(ahead)) { load(ahead, ra[j], rb[j]); advance(ahead); }
                    if (!warp_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, p.timeout_ns, lane)) {
                        aborted = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t slot = sf_base + static_cast<uint32_t>(stage) * SF_STRIDE;
                    tmem_st_32x32b_x4(slot, wa0, wa1, wa2, wa3);
                    tmem_st_32x32b_x4(slot + 4, wb0, wb0, wb0, wb0);
                    if (BN == 256) tmem_st_32x32b_x4(slot + 8, wb1, wb1, wb1, wb1);
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[stage]);
                    if (stage == STAGES - 1) phase ^= 1u;
                    advance(cur);
                }
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

template <int BN, bool OUT_FP8>
cudaError_t launch_bn(const GemmArgs& a, cudaStream_t st) {
    TcParams p;
    if (!fill_params(p, a, 1, BN, kWaitTimeoutNs, OUT_FP8 ? 1 : 2)) return cudaErrorInvalidValue;
    p.sf_vec = 1;
    for (int gi = 0; gi < 2; ++gi) {
        const GemmGroup& g = a.g[gi];
        if (g.n_mats == 0) continue;
        const bool aligned = (reinterpret_cast<uintptr_t>(g.a_scales) % 16 == 0) &&
                             (reinterpret_cast<uintptr_t>(g.b_scales) % 16 == 0);
        if (g.K % (4 * BK) != 0 || !aligned) p.sf_vec = 0;
    }
    constexpr int smem = FCfg<BN>::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory budget");
    auto kernel = grouped_ffn_fp8_kernel<BN, OUT_FP8>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, dim3(device_sm_count()), dim3(NUM_THREADS), smem, st, 1, p);
}

}  // namespace

// Weight tiles are 256 wide.  128-wide tiles (FCfg<128>) double the tile
// count on decode-sized batches, which evens out the last wave, but measured
// slower on the V3 decode batch (0.293 against 0.269 ms): the per-stage cost
// of the block-scaled MMA is nearly the same at N = 128 as at N = 256.  A
// 224-wide second layer (d_model = 7168 = 32 x 224; two disjoint accumulators
// and the scale slots fill the 512 columns, so no tile waits for the
// previous one's overlapping columns; weight scales picked per row, since a
// tile then starts inside a 128-row block) passed parity but measured slower
// on the V3 prefill layer (2.26 against 2.07 ms, same box): the extra tiles
// cost more than the overlap wait they remove.  Eight epilogue warps for the
// second layer (two per lane quadrant, 448 threads, which caps registers at
// 128 with spills) also measured slower (2.36 against 2.23 ms, same box), and
// 128-wide first-layer tiles for the decode batch alone (twice the tiles of
// its 2.5 waves) gained nothing (0.325 against 0.324 ms).  An L2 prefetch
// (cp.async.bulk.prefetch.tensor) of the A and B boxes 4, 8 or 16 items ahead
// of the ring's loads made the V3 prefill layer slower, the more so the
// further ahead (2.05 against 2.71, 2.85 and 3.17 ms, same box).  Separate
// rings for A (2 stages, loaded by a scale-factor warp after the same wait
// as its scale slot) and B (5 stages: 128 KB of weights in flight instead of
// 96) passed parity but measured slower (2.39 against 2.02 ms; with 4 + 4
// stages 2.10): the A tile then reaches the MMA too late.
cudaError_t launch_grouped_ffn_fp8(const Dims&, const GemmArgs& a, cudaStream_t st) {
    return a.out_fp8 ? launch_bn<256, true>(a, st) : launch_bn<256, false>(a, st);
}

}  // namespace moe

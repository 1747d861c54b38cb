// Pieces shared by the tensor-core grouped-GEMM kernels (bf16 and FP8):
// kernel parameters, the per-CTA segment table built from the device-side
// dispatch offsets, tile decoding, and the host-side parameter fill.
//
// Segments: one per routed expert (rows offsets[e] .. offsets[e+1]-1 of A
// and C; with a segment map, segment i holds rows of expert seg_mat[i]), then
// one per shared expert (fixed_rows rows each).  A segment of
// `rows` rows has ceil(rows/128) m-tiles and ceil(N/BN) n-tiles; its tiles are
// numbered n-tile-major with m fastest, so CTAs that run at the same time
// work on the same weight tile.
#pragma once

#include <cuda.h>
#include <cstring>
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace ffn {

constexpr int BM = 128;
constexpr int MAX_SEGS = 256 + 8;

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
    int a_rows;
    const int32_t* seg_mat;   // routed: weight matrix of each segment, or nullptr
    int n_weights;            // matrices seg_mat may name
};

struct __align__(64) TcParams {
    CUtensorMap a_map[2];
    CUtensorMap b_map[2];
    CUtensorMap c_map[2];     // outputs, for TMA stores (FP8 engine)
    GroupDev g[2];
    int silu;
    int out_fp8;
    int sf_vec;               // FP8: scales read as float4 over four k-blocks
    int32_t* status;
    uint64_t timeout_ns;
};

struct TileInfo {
    int grp, mat, rows_left, a_row, c_row, n0, kblocks;
};

// Segment table in shared memory (SEG_INTS ints).
struct SegTable {
    int* start;   // MAX_SEGS + 1: first tile of each segment, start[nseg] = total
    int* rows;
    int* arow;
    int* crow;
    int* mat;     // group << 16 | matrix index
    static constexpr int SEG_INTS = (MAX_SEGS + 1) + 4 * MAX_SEGS;
    __device__ explicit SegTable(int* base)
        : start(base), rows(base + MAX_SEGS + 1), arow(rows + MAX_SEGS), crow(arow + MAX_SEGS),
          mat(crow + MAX_SEGS) {}
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Builds the table cooperatively (all threads of the block call it; ends with
// the scan done by warp 0 -- the caller synchronises afterwards).  A
// scheduled tile covers MGROUP consecutive m-tiles (2 for CTA pairs).
template <int BN, int MGROUP = 1>
__device__ __forceinline__ int build_seg_table(const TcParams& p, SegTable& t, int nthreads) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n0segs = p.g[0].n_mats, n1segs = p.g[1].n_mats;
    const int nseg = n0segs + n1segs;
    for (int s = tid; s < nseg; s += nthreads) {
        int rows, arow, crow, packed, N;
        if (s < n0segs) {
            const GroupDev& g = p.g[0];
            const int o0 = g.offsets[s], o1 = g.offsets[s + 1];
            rows = o1 - o0;
            if (g.seg_mat) {
                // caller-made segments: one out of bounds, or naming no
                // matrix, is skipped and reported
                const int m = g.seg_mat[s];
                if (o0 < 0 || rows < 0 || o1 > g.a_rows || m < 0 || m >= g.n_weights) {
                    rows = 0;
                    set_device_status(p.status, MOE_DEV_BAD_ROUTING);
                }
            }
            arow = g.a_row_base + o0;
            crow = g.c_row_base + o0;
            packed = g.seg_mat ? g.seg_mat[s] : s;     // the segment's weight matrix
            N = g.N;
        } else {
            const GroupDev& g = p.g[1];
            const int i = s - n0segs;
            rows = g.fixed_rows;
            arow = g.a_row_base + i * g.a_seg_stride;
            crow = g.c_row_base + i * g.fixed_rows;
            packed = (1 << 16) | i;
            N = g.N;
        }
        t.rows[s] = rows;
        t.arow[s] = arow;
        t.crow[s] = crow;
        t.mat[s] = packed;
        t.start[s + 1] = ceil_div(ceil_div(rows, BM), MGROUP) * ceil_div(N, BN);   // tile count, scanned below
    }
    __syncthreads();
    if (warp == 0) {                                                // inclusive scan of tile counts
        int carry = 0;
        for (int base = 0; base < nseg; base += 32) {
            const int i = base + lane;
            int v = (i < nseg) ? t.start[i + 1] : 0;
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

// Tile `tile` of the table; with MGROUP > 1 the m-tile is MGROUP * group + sub
// (rows_left <= 0 when that m-tile lies past the segment's end).
template <int BN, int BK, int MGROUP = 1>
__device__ __forceinline__ TileInfo decode_tile(int tile, const TcParams& p, const SegTable& t, int nseg,
                                                int sub = 0) {
    int lo = 0, hi = nseg - 1;                      // last s with start[s] <= tile
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (t.start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int s = lo;
    const int local = tile - t.start[s];
    const int mgroups = ceil_div(ceil_div(t.rows[s], BM), MGROUP);
    const int nt = local / mgroups, mt = (local % mgroups) * MGROUP + sub;
    TileInfo ti;
    ti.grp = t.mat[s] >> 16;
    ti.mat = t.mat[s] & 0xFFFF;
    ti.rows_left = t.rows[s] - mt * BM;
    ti.a_row = t.arow[s] + mt * BM;
    ti.c_row = t.crow[s] + mt * BM;
    ti.n0 = nt * BN;
    ti.kblocks = ceil_div(p.g[ti.grp].K, BK);
    return ti;
}

// Bounded wait done by lane 0 only; the result is broadcast so that the warp
// leaves converged (tcgen05.ld / tcgen05.st that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, uint64_t timeout_ns, int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(bar, parity, abort_flag, status, timeout_ns) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Host: fills the parameter block of both groups; elem = operand bytes,
// bn = weight rows per tile, out_elem > 0: also the output maps for TMA
// stores of 64-byte x 32-row boxes (out_elem = output element bytes).
// Returns false if a tensor map cannot be encoded.
inline bool fill_params(TcParams& p, const GemmArgs& a, int elem, int bn, uint64_t timeout_ns, int out_elem = 0) {
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
        d.a_rows = g.a_rows;
        d.seg_mat = g.seg_mat;
        d.n_weights = g.n_weights > 0 ? g.n_weights : g.n_mats;
        if (!encode_tma_2d(&p.a_map[gi], g.A, g.a_rows, g.K, elem, BM)) return false;
        if (!encode_tma_3d(&p.b_map[gi], g.B, g.n_weights > 0 ? g.n_weights : g.n_mats, g.N, g.K, elem, bn))
            return false;
        if (out_elem > 0 && !encode_tma_2d_store64(&p.c_map[gi], g.C, g.c_rows, g.N, out_elem, 32)) return false;
    }
    p.silu = a.silu;
    p.out_fp8 = a.out_fp8;
    p.status = a.status;
    p.timeout_ns = timeout_ns;
    return true;
}

}  // namespace ffn
}  // namespace moe

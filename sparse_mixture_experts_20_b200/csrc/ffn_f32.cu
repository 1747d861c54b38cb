// fp32 grouped expert FFN (MOE_F32 mode) on the CUDA cores.
//
// "論文解説: DeepSeekMoE" §アルゴリズム: expert = Linear(d, d_ff) + bias ->
// SiLU -> Linear(d_ff, d) + bias.  fp32 activations and weights need fp32
// arithmetic end to end (the tensor cores' tf32 path would lose precision),
// so this engine is a tiled SIMT GEMM: 64x64 output tiles, 256 threads with
// 4x4 register blocks, K staged through shared memory 16 columns at a time.
// Segments (one per routed expert, rows from the device-side offsets, then
// one per shared expert) are walked the same way as in the tensor-core
// engine; rows past a segment's end are loaded as zeros and never stored.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int FBM = 64, FBN = 64, FBK = 16;
constexpr int MAX_SEGS = 256 + 8;

struct F32Group {
    int n_mats;
    const int32_t* offsets;
    const int32_t* seg_mat;   // routed: weight matrix of each segment, or nullptr
    int fixed_rows;
    const float* A;
    int a_rows;
    int a_row_base, a_seg_stride;
    const float* B;
    const float* bias;
    float* C;
    int c_row_base;
    int N, K;
};

struct F32Params {
    F32Group g[2];
    int silu;
    int n_weights;            // matrices the routed segment map may name
    int32_t* status;
};

__global__ void __launch_bounds__(256)
ffn_f32_kernel(const __grid_constant__ F32Params p) {
    __shared__ int seg_start[MAX_SEGS + 1];
    __shared__ int seg_rows[MAX_SEGS];
    __shared__ float As[FBK][FBM + 4];
    __shared__ float Bs[FBK][FBN + 4];
    pdl_wait();
    pdl_allow_next();
    const int tid = threadIdx.x;
    const int n0segs = p.g[0].n_mats, nseg = n0segs + p.g[1].n_mats;
    for (int s = tid; s < nseg; s += 256) {
        int rows = (s < n0segs) ? p.g[0].offsets[s + 1] - p.g[0].offsets[s] : p.g[1].fixed_rows;
        if (s < n0segs && p.g[0].seg_mat) {
            // caller-made segments: one out of bounds, or naming no matrix,
            // is skipped and reported
            const int o0 = p.g[0].offsets[s], m = p.g[0].seg_mat[s];
            if (o0 < 0 || rows < 0 || o0 + rows > p.g[0].a_rows || m < 0 || m >= p.n_weights) {
                rows = 0;
                if (blockIdx.x == 0 && blockIdx.y == 0) set_device_status(p.status, MOE_DEV_BAD_ROUTING);
            }
        }
        seg_rows[s] = rows;
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int s = 0; s < nseg; ++s) { seg_start[s] = run; run += (seg_rows[s] + FBM - 1) / FBM; }
        seg_start[nseg] = run;
    }
    __syncthreads();
    const int mt_global = blockIdx.x;
    if (mt_global >= seg_start[nseg]) return;
    int s = 0;
    while (seg_start[s + 1] <= mt_global) ++s;
    const int grp = s < n0segs ? 0 : 1;
    const F32Group& g = p.g[grp];
    const int mat = grp == 0 ? s : s - n0segs;
    const int mt = mt_global - seg_start[s];
    const int rows_left = seg_rows[s] - mt * FBM;
    int a_row, c_row;
    if (grp == 0) {
        a_row = g.a_row_base + g.offsets[mat] + mt * FBM;
        c_row = g.c_row_base + g.offsets[mat] + mt * FBM;
    } else {
        a_row = g.a_row_base + mat * g.a_seg_stride + mt * FBM;
        c_row = g.c_row_base + mat * g.fixed_rows + mt * FBM;
    }
    const int n0 = blockIdx.y * FBN;
    if (n0 >= g.N) return;
    const int wmat = (grp == 0 && g.seg_mat) ? g.seg_mat[mat] : mat;    // the segment's weights
    const float* Bm = g.B + static_cast<size_t>(wmat) * g.N * g.K;

    const int ty = tid / 16, tx = tid % 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < g.K; k0 += FBK) {
        for (int e = tid; e < FBM * FBK; e += 256) {
            const int r = e / FBK, c = e % FBK;
            As[c][r] = (r < rows_left && k0 + c < g.K) ? g.A[static_cast<size_t>(a_row + r) * g.K + k0 + c] : 0.f;
            const int n = n0 + r;
            Bs[c][r] = (n < g.N && k0 + c < g.K) ? Bm[static_cast<size_t>(n) * g.K + k0 + c] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < FBK; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { av[i] = As[kk][ty * 4 + i]; bv[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
        if (r >= rows_left) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= g.N) continue;
            float v = acc[i][j] + g.bias[static_cast<size_t>(wmat) * g.N + n];
            if (p.silu) v = v / (1.0f + expf(-v));
            g.C[static_cast<size_t>(c_row + r) * g.N + n] = v;
        }
    }
}

}  // namespace

cudaError_t launch_grouped_ffn_f32(const Dims& dm, const GemmArgs& a, cudaStream_t st) {
    F32Params p{};
    int ntiles = 1;
    for (int gi = 0; gi < 2; ++gi) {
        const GemmGroup& s = a.g[gi];
        F32Group& d = p.g[gi];
        d.n_mats = s.n_mats;
        if (s.n_mats == 0) continue;
        d.offsets = s.offsets;
        d.seg_mat = s.seg_mat;
        d.fixed_rows = s.fixed_rows;
        d.A = static_cast<const float*>(s.A);
        d.a_rows = s.a_rows;
        d.a_row_base = s.a_row_base;
        d.a_seg_stride = s.a_seg_stride;
        d.B = static_cast<const float*>(s.B);
        d.bias = s.bias;
        d.C = static_cast<float*>(s.C);
        d.c_row_base = s.c_row_base;
        d.N = s.N;
        d.K = s.K;
        ntiles = max(ntiles, (s.N + FBN - 1) / FBN);
    }
    p.silu = a.silu;
    p.n_weights = a.g[0].n_weights > 0 ? a.g[0].n_weights : a.g[0].n_mats;
    p.status = a.status;
    // m-tiles: at most one per 64 rows of the routed rows plus one per segment
    // (its ragged tail), and those of the fixed segments
    int mt_bound = 0;
    if (a.g[0].n_mats > 0) mt_bound += (a.g[0].a_rows + FBM - 1) / FBM + a.g[0].n_mats;
    if (a.g[1].n_mats > 0) mt_bound += a.g[1].n_mats * ((a.g[1].fixed_rows + FBM - 1) / FBM);
    if (mt_bound < 1) mt_bound = 1;
    (void)dm;
    return launch_pdl(ffn_f32_kernel, dim3(mt_bound, ntiles), dim3(256), 0, st, 1, p);
}

}  // namespace moe

// GPU executor of the layer backward.
//
// fp32 layers: each step of bwd::run_backward (backward.cuh) runs as one
// grid-stride kernel of 256 threads, one output element per iteration.
//
// bf16 layers: the router and gate steps are the same fixed-order functors
// (the gate gradients one warp per slot); every expert GEMM runs on the
// tensor cores (bwd_gemm.cu) over padded row segments:
//   1. poff: each routed expert's row count rounded up to 16, scanned;
//   2. padded rows: x_p[pr] = x_disp[r], dy_p[pr] = g * dout[t] (bf16), zero
//      rows in each expert's padding;
//   3. recompute  z = x_p W1^T + b1          -> SiLU(z), SiLU'(z)  (bf16)
//   4. dgrad      dz = (dy_p W2) * SiLU'(z)  -> bf16
//   5. dgrad      dx rows = dz W1            -> fp32
//   6. wgrad      dW2 = dy_p^T SiLU(z), dW1 = dz^T x_p (fp32, contraction
//      over each expert's padded rows; the padding rows are zero in dy_p and
//      dz, so they add nothing)
//   shared experts in the same launches (rows = the T tokens, dy = dout; the
//   shared hidden activations of all shared experts side by side in one
//   (T, n_shared * d_ff_shared) matrix, so dx and dW1 of all shared experts
//   are one GEMM each);
//   7. bias gradients: column sums in two fixed-order passes (16-row chunk
//      partials -- for dy made by the padding kernel as it writes dy -- then
//      the chunks of each segment in order);
//   8. dx = router part + shared part + the kept slots' rows (+ g * dout for
//      slots passed through).
// Every reduction has a fixed order: the result is bit-reproducible.
#include <algorithm>
#include <cstring>
#include "backward.cuh"

namespace moe {
namespace {

template <class F>
__global__ void __launch_bounds__(256) for_each_kernel(size_t n, F f) {
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        f(i);
}

struct GpuExec {
    cudaStream_t st;
    cudaError_t err;
    int launches;
    int max_blocks;
    template <class F> void run(size_t n, const F& f) {
        if (err != cudaSuccess || n == 0) return;
        size_t blocks = (n + 255) / 256;
        if (blocks > static_cast<size_t>(max_blocks)) blocks = max_blocks;   // then the loop strides
        for_each_kernel<F><<<static_cast<unsigned>(blocks), 256, 0, st>>>(n, f);
        ++launches;
        err = cudaGetLastError();
    }
};

// ------------------------------------------------------------ bf16 path

// a[slot] = <dout_t, y_row> (kept), <dout_t, x_t> (passed through), else 0:
// one warp per slot, 16-byte loads, lanes own fixed column chunks, fixed
// butterfly order.
template <typename XT>
__global__ void __launch_bounds__(256) gate_grad_warp_kernel(int TK, int K, int d, int passthrough,
                                                              const int32_t* slot_row, const XT* dout,
                                                              const XT* y, const XT* x, float* a) {
    constexpr int V = 16 / sizeof(XT);
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int slot = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); slot < TK; slot += warps) {
        const int t = slot / K;
        const int row = slot_row[slot];
        const XT* other = row >= 0 ? y + static_cast<size_t>(row) * d
                                   : ((row == -1 && passthrough) ? x + static_cast<size_t>(t) * d : nullptr);
        float acc = 0.f;
        if (other) {
            const XT* dr = dout + static_cast<size_t>(t) * d;
            for (int c = lane * V; c < d; c += 32 * V) {
                const uint4 pa = *reinterpret_cast<const uint4*>(dr + c);
                const uint4 pb = *reinterpret_cast<const uint4*>(other + c);
                const XT* ea = reinterpret_cast<const XT*>(&pa);
                const XT* eb = reinterpret_cast<const XT*>(&pb);
#pragma unroll
                for (int j = 0; j < V; ++j) acc += bwd::ld(ea, j) * bwd::ld(eb, j);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) a[slot] = acc;
    }
}

// dl[t][j] = dJ/dl of token t (softmax of its logits, the gates' and the
// balance loss's share of ds), one warp per token, lanes over experts; also
// the bf16 copy dl_b (row stride Epad, zero columns E .. Epad-1) that the
// tensor-core router gradients read.  Reductions in fixed butterfly order.
__global__ void __launch_bounds__(256) router_grad_warp_kernel(int T, int E, int K, int Epad, float bal,
                                                                const float* logits, const int32_t* topk_idx,
                                                                const float* gates, const float* a,
                                                                const int32_t* counts, float* dl,
                                                                __nv_bfloat16* dl_b) {
    constexpr int JMAX = 8;                          // E <= 256
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
        const float* l = logits + static_cast<size_t>(t) * E;
        float lv[JMAX];
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < JMAX; ++i) {
            const int j = lane + 32 * i;
            lv[i] = j < E ? l[j] : -INFINITY;
            m = fmaxf(m, lv[i]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float z = 0.f;
#pragma unroll
        for (int i = 0; i < JMAX; ++i) {
            lv[i] = (lane + 32 * i) < E ? expf(lv[i] - m) : 0.f;
            z += lv[i];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
        // S = sum of s over the chosen experts; common = sum_k a_k g_k (same order on every lane)
        float S = 0.f, common = 0.f;
        for (int k = 0; k < K; ++k) {
            const int j = topk_idx[static_cast<size_t>(t) * K + k];
            if (j >= 0 && j < E) S += expf(l[j] - m) / z;
            common += a[static_cast<size_t>(t) * K + k] * gates[static_cast<size_t>(t) * K + k];
        }
        float ds[JMAX];
        float sds = 0.f;
#pragma unroll
        for (int i = 0; i < JMAX; ++i) {
            const int j = lane + 32 * i;
            float v = 0.f;
            if (j < E) {
                v = bal * static_cast<float>(counts[j]);
                for (int k = 0; k < K; ++k)
                    if (topk_idx[static_cast<size_t>(t) * K + k] == j) v += (a[static_cast<size_t>(t) * K + k] - common) / S;
                lv[i] = lv[i] / z;                   // s_j
            }
            ds[i] = v;
            sds += lv[i] * v;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sds += __shfl_xor_sync(0xffffffffu, sds, off);
#pragma unroll
        for (int i = 0; i < JMAX; ++i) {
            const int j = lane + 32 * i;
            if (j < E) {
                const float v = lv[i] * (ds[i] - sds);
                dl[static_cast<size_t>(t) * E + j] = v;
                dl_b[static_cast<size_t>(t) * Epad + j] = __float2bfloat16_rn(v);
            } else if (j < Epad) {
                dl_b[static_cast<size_t>(t) * Epad + j] = __float2bfloat16_rn(0.f);
            }
        }
    }
}

__global__ void __launch_bounds__(256) f32_to_bf16_kernel(size_t n, const float* in, __nv_bfloat16* out) {
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        out[i] = __float2bfloat16_rn(in[i]);
}

// out[i] = sum over s of part[s * n + i], in split order.
__global__ void __launch_bounds__(256) sum_splits_kernel(size_t n, int splits, const float* part, float* out) {
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        float acc = 0.f;
        for (int s2 = 0; s2 < splits; ++s2) acc += part[static_cast<size_t>(s2) * n + i];
        out[i] = acc;
    }
}

// part[ch][c] = sum of rows ch*CH .. of column c of an fp32 (rows, ncols)
// matrix (any ncols); one column per thread.
template <int CH>
__global__ void __launch_bounds__(256) colsum_chunks_f32_kernel(const float* M, int ncols, int n_rows, float* part) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= ncols) return;
    for (int ch = blockIdx.y; ch * CH < n_rows; ch += gridDim.y) {
        const int r0 = ch * CH, r1 = min(r0 + CH, n_rows);
        float acc = 0.f;
        for (int r = r0; r < r1; ++r) acc += M[static_cast<size_t>(r) * ncols + c];
        part[static_cast<size_t>(ch) * ncols + c] = acc;
    }
}

// poff[e] = sum over e' < e of roundup16(offsets[e'+1] - offsets[e']);
// also clears the status word.  One warp.
__global__ void pad_offsets_kernel(const int32_t* offsets, int E, int32_t* poff, int32_t* status) {
    const int lane = threadIdx.x;
    if (lane == 0) *status = 0;
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
        const int e = base + lane;
        int v = e < E ? ((offsets[e + 1] - offsets[e] + 15) & ~15) : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += o;
        }
        if (e < E) poff[e + 1] = v + carry;
        carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) poff[0] = 0;
}

// Padded rows in chunks of 16 (the padding unit, so a chunk lies in one
// expert's segment): x_p[pr] = x_disp[r], dy_p[pr] = g * dout[t] (bf16) for
// the rows of a segment, zeros in its padding, and the chunk's column sums
// of dy_p as stored (part[ch][c], the first pass of db2).  Block = (a slab
// of 2048 columns, a chunk); thread = 8 columns; the 16 rows' sources are
// looked up once per chunk.
__global__ void __launch_bounds__(256) pad_rows_kernel(int E, int K, int d, const int32_t* offsets,
                                                       const int32_t* poff, const int32_t* row_slot,
                                                       const float* gates, const __nv_bfloat16* dout,
                                                       const __nv_bfloat16* x_disp, __nv_bfloat16* x_p,
                                                       __nv_bfloat16* dy_p, float* part) {
    __shared__ int s_r[16], s_t[16];
    __shared__ float s_g[16];
    const int total = poff[E];
    const int c = 8 * (blockIdx.x * blockDim.x + threadIdx.x);
    for (int ch = blockIdx.y; ch * 16 < total; ch += gridDim.y) {
        if (threadIdx.x < 16) {
            const int pr = ch * 16 + threadIdx.x;
            int lo = 0, hi = E - 1;                     // last e with poff[e] <= pr
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (poff[mid] <= pr) lo = mid; else hi = mid - 1;
            }
            const int i = pr - poff[lo];
            int r = -1, t = 0;
            float g = 0.f;
            if (i < offsets[lo + 1] - offsets[lo]) {
                r = offsets[lo] + i;
                const int slot = row_slot[r];
                t = slot / K;
                g = gates[slot];
            }
            s_r[threadIdx.x] = r;
            s_t[threadIdx.x] = t;
            s_g[threadIdx.x] = g;
        }
        __syncthreads();
        if (c < d) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int i = 0; i < 16; ++i) {
                const size_t pr = static_cast<size_t>(ch) * 16 + i;
                const int r = s_r[i];
                uint4 xv = make_uint4(0u, 0u, 0u, 0u), yv = make_uint4(0u, 0u, 0u, 0u);
                if (r >= 0) {
                    xv = *reinterpret_cast<const uint4*>(x_disp + static_cast<size_t>(r) * d + c);
                    yv = *reinterpret_cast<const uint4*>(dout + static_cast<size_t>(s_t[i]) * d + c);
                    const float g = s_g[i];
                    uint32_t* w = reinterpret_cast<uint32_t*>(&yv);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
                        const __nv_bfloat162 o = __floats2bfloat162_rn(g * f.x, g * f.y);
                        const float2 q = __bfloat1622float2(o);
                        acc[2 * j] += q.x;
                        acc[2 * j + 1] += q.y;
                        w[j] = *reinterpret_cast<const uint32_t*>(&o);
                    }
                }
                *reinterpret_cast<uint4*>(x_p + pr * d + c) = xv;
                *reinterpret_cast<uint4*>(dy_p + pr * d + c) = yv;
            }
            float4* po = reinterpret_cast<float4*>(part + static_cast<size_t>(ch) * d + c);
            po[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            po[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        __syncthreads();
    }
}

// part[ch][c] = sum of rows ch*CH .. min(ch*CH + CH, n_rows) - 1 of column c
// (bf16 matrix, row stride ld); n_rows from *n_rows_dev when given.
template <int CH>
__global__ void __launch_bounds__(256) colsum_chunks_kernel(const __nv_bfloat16* M, int ld, int ncols,
                                                            const int32_t* n_rows_dev, int n_rows, float* part) {
    const int rows = n_rows_dev ? *n_rows_dev : n_rows;
    const int c = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (c >= ncols) return;
    for (int ch = blockIdx.y; ch * CH < rows; ch += gridDim.y) {
        const int r0 = ch * CH, r1 = min(r0 + CH, rows);
        float s0 = 0.f, s1 = 0.f;
        for (int r = r0; r < r1; ++r) {
            const float2 f = __bfloat1622float2(
                *reinterpret_cast<const __nv_bfloat162*>(M + static_cast<size_t>(r) * ld + c));
            s0 += f.x;
            s1 += f.y;
        }
        *reinterpret_cast<float2*>(part + static_cast<size_t>(ch) * ncols + c) = make_float2(s0, s1);
    }
}

// out[copy * copy_stride + s * ncols + c] = sum over the chunks of segment s
// of part[ch][c], in chunk order.  Segment s spans rows seg[s] .. seg[s+1]-1
// (multiples of CH) or, with seg == nullptr, rows 0 .. fixed_rows-1.  Block =
// (32 columns, a segment): warp w sums the w-th of 8 contiguous runs of the
// segment's chunks (lane = column), then the 8 run sums are added in run order.
template <int CH>
__global__ void __launch_bounds__(256) colsum_segments_kernel(const float* part, int ncols, const int32_t* seg,
                                                              int nseg, int fixed_rows, float* out, int copies,
                                                              int copy_stride) {
    __shared__ float sm[8][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int s = blockIdx.y, c = blockIdx.x * 32 + lane;
    const int ch0 = seg ? seg[s] / CH : 0;
    const int ch1 = seg ? seg[s + 1] / CH : (fixed_rows + CH - 1) / CH;
    const int per = (ch1 - ch0 + 7) / 8;
    const int a = ch0 + warp * per, b = min(ch1, a + per);
    float acc = 0.f;
    if (c < ncols)
        for (int ch = a; ch < b; ++ch) acc += part[static_cast<size_t>(ch) * ncols + c];
    sm[warp][lane] = acc;
    __syncthreads();
    if (warp == 0 && c < ncols) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += sm[w][lane];
        for (int k = 0; k < copies; ++k) out[static_cast<size_t>(k) * copy_stride + static_cast<size_t>(s) * ncols + c] = t;
    }
    (void)nseg;
}

// dx[t][c] = dx_router[t][c] + dx_shared[t][c] + sum_k (kept: the bf16 dx
// row of the slot's padded row; passed through: g * dout[t][c]), one warp per
// token: the slots' rows are looked up once, lanes take 8 columns at a time.
__global__ void __launch_bounds__(256) dx_final_kernel(int T, int K, int d, int passthrough, const float* dx_router,
                                                       const float* dx_shared, const int32_t* slot_row,
                                                       const int32_t* topk_idx, const int32_t* offsets,
                                                       const int32_t* poff, const float* gates,
                                                       const __nv_bfloat16* dxr_p, const __nv_bfloat16* dout,
                                                       float* dx) {
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
        // lane k < K: padded row of slot k (>= 0), -1 passed through, -2 nothing
        long long my_row = -2;
        float my_g = 0.f;
        if (lane < K) {
            const int row = slot_row[static_cast<size_t>(t) * K + lane];
            if (row >= 0) {
                const int e = topk_idx[static_cast<size_t>(t) * K + lane];
                my_row = row - offsets[e] + poff[e];
            } else if (row == -1 && passthrough) {
                my_row = -1;
                my_g = gates[static_cast<size_t>(t) * K + lane];
            }
        }
        const size_t base = static_cast<size_t>(t) * d;
        for (int c = lane * 8; c < d; c += 256) {
            float v[8];
            const float4 r0 = *reinterpret_cast<const float4*>(dx_router + base + c);
            const float4 r1 = *reinterpret_cast<const float4*>(dx_router + base + c + 4);
            v[0] = r0.x; v[1] = r0.y; v[2] = r0.z; v[3] = r0.w; v[4] = r1.x; v[5] = r1.y; v[6] = r1.z; v[7] = r1.w;
            if (dx_shared) {
                const float4 s0 = *reinterpret_cast<const float4*>(dx_shared + base + c);
                const float4 s1 = *reinterpret_cast<const float4*>(dx_shared + base + c + 4);
                v[0] += s0.x; v[1] += s0.y; v[2] += s0.z; v[3] += s0.w;
                v[4] += s1.x; v[5] += s1.y; v[6] += s1.z; v[7] += s1.w;
            }
            for (int k = 0; k < K; ++k) {
                const long long row = __shfl_sync(0xffffffffu, my_row, k);
                const float gk = __shfl_sync(0xffffffffu, my_g, k);
                if (row == -2) continue;
                const __nv_bfloat16* src = row >= 0 ? dxr_p + static_cast<size_t>(row) * d + c : dout + base + c;
                const float w = row >= 0 ? 1.f : gk;
                const uint4 q = *reinterpret_cast<const uint4*>(src);
                const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qw[j]));
                    v[2 * j] += w * f.x;
                    v[2 * j + 1] += w * f.y;
                }
            }
            *reinterpret_cast<float4*>(dx + base + c) = make_float4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<float4*>(dx + base + c + 4) = make_float4(v[4], v[5], v[6], v[7]);
        }
    }
}

struct TcLayout {
    size_t status, a, dl, dl_b, w_rb, rw_part, dxacc, poff, x_p, dy_p, h_p, sp_p, dz_p, dxr_p, h_s, sp_s, dz_s,
        dx_s, part, total;
    int rows_cap;   // padded routed rows
    int epad;       // row stride of dl_b
    int rw_splits;  // token splits of the router weight gradient
    int rw_chunk;   // tokens per split
};

// The router weight gradient (M = N_r, N = d, K = T) has few output tiles:
// its tokens are split so that about this many tiles run at once (a fixed
// number, so that the workspace and the summation order do not depend on
// the device).
constexpr int kRouterSplitTiles = 296;

constexpr int kChunkRouted = 16;    // row chunk of the routed column sums (the padding unit)
constexpr int kChunkShared = 16;     // row chunk of the token-wide column sums

TcLayout tc_layout(const Dims& dm) {
    TcLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + 255) & ~static_cast<size_t>(255);
        return o;
    };
    const size_t T = dm.T, d = dm.d, E = dm.E, K = dm.K, dff = dm.dff;
    const size_t sw = static_cast<size_t>(dm.S) * dm.dffs;
    const size_t Rp = (static_cast<size_t>(dm.r_cap) + 15 * E + 15) & ~static_cast<size_t>(15);
    L.rows_cap = static_cast<int>(Rp);
    L.epad = static_cast<int>((E + 7) & ~static_cast<size_t>(7));
    {
        const int tiles = static_cast<int>(((E + 127) / 128) * ((d + 255) / 256));
        int splits = (kRouterSplitTiles + tiles - 1) / tiles;
        const int max_splits = (dm.T + 255) / 256;
        if (splits > max_splits) splits = max_splits;
        if (splits < 1) splits = 1;
        const int chunk = ((dm.T + splits - 1) / splits + 15) & ~15;
        L.rw_chunk = chunk;
        L.rw_splits = (dm.T + chunk - 1) / chunk;
    }
    L.status = take(256);
    L.a = take(T * K * 4);
    L.dl = take(T * E * 4);
    L.dl_b = take(T * static_cast<size_t>(L.epad) * 2);
    L.w_rb = take(E * d * 2);
    L.rw_part = take(L.rw_splits > 1 ? static_cast<size_t>(L.rw_splits) * E * d * 4 : 0);
    L.dxacc = take(T * d * 4);
    L.poff = take((E + 1) * 4);
    L.x_p = take(Rp * d * 2);
    L.dy_p = take(Rp * d * 2);
    L.h_p = take(Rp * dff * 2);
    L.sp_p = take(Rp * dff * 2);
    L.dz_p = take(Rp * dff * 2);
    L.dxr_p = take(Rp * d * 2);
    L.h_s = take(T * sw * 2);
    L.sp_s = take(T * sw * 2);
    L.dz_s = take(T * sw * 2);
    L.dx_s = take(sw ? T * d * 4 : 0);
    const size_t pr = (Rp / kChunkRouted) * (d > dff ? d : dff);
    size_t ps = ((T + kChunkShared - 1) / kChunkShared) * (d > sw ? d : sw);
    if (((T + kChunkShared - 1) / kChunkShared) * E > ps) ps = ((T + kChunkShared - 1) / kChunkShared) * E;
    L.part = take((pr > ps ? pr : ps) * 4);
    L.total = off;
    return L;
}

BwdGemmGroup group0() {
    BwdGemmGroup g;
    std::memset(&g, 0, sizeof(g));
    return g;
}

cudaError_t run_backward_bf16(const Dims& dm, float lam, const moe_backward_io& io, void* bws, cudaStream_t st,
                              int& launches) {
    using bf = __nv_bfloat16;
    const TcLayout L = tc_layout(dm);
    uint8_t* base = static_cast<uint8_t*>(bws);
    auto F = [&](size_t o) { return reinterpret_cast<float*>(base + o); };
    auto B = [&](size_t o) { return reinterpret_cast<bf*>(base + o); };
    int32_t* status = reinterpret_cast<int32_t*>(base + L.status);
    int32_t* poff = reinterpret_cast<int32_t*>(base + L.poff);
    float *a = F(L.a), *dl = F(L.dl), *dxacc = F(L.dxacc), *dx_s = F(L.dx_s), *part = F(L.part);
    float* rw_part = F(L.rw_part);
    bf *dl_b = B(L.dl_b), *w_rb = B(L.w_rb), *dxr_p = B(L.dxr_p);
    bf *x_p = B(L.x_p), *dy_p = B(L.dy_p), *h_p = B(L.h_p), *sp_p = B(L.sp_p), *dz_p = B(L.dz_p);
    bf *h_s = B(L.h_s), *sp_s = B(L.sp_s), *dz_s = B(L.dz_s);
    const int T = dm.T, d = dm.d, E = dm.E, K = dm.K, dff = dm.dff, S = dm.S, dffs = dm.dffs, Rp = L.rows_cap;
    const int sw = S * dffs;
    const bf* x = static_cast<const bf*>(io.x);
    const bf* dout = static_cast<const bf*>(io.dout);
    const int sms = device_sm_count();
    GpuExec ex{st, cudaSuccess, 0, sms * 16};
    auto check = [&](cudaError_t e) { if (ex.err == cudaSuccess && e != cudaSuccess) ex.err = e; };

    // router and gates
    pad_offsets_kernel<<<1, 32, 0, st>>>(io.offsets, E, poff, status);
    check(cudaGetLastError());
    ++ex.launches;
    {
        const int TK = T * K;
        const int blocks = std::min((TK + 7) / 8, sms * 8);
        gate_grad_warp_kernel<bf><<<blocks, 256, 0, st>>>(TK, K, d, dm.passthrough, io.slot_row, dout,
                                                         static_cast<const bf*>(io.y), x, a);
        check(cudaGetLastError());
        ++ex.launches;
    }
    const float bal = lam * dm.alpha * static_cast<float>(dm.E) /
                      (static_cast<float>(dm.T) * static_cast<float>(dm.T) * static_cast<float>(dm.K));
    {
        const int blocks = std::min((T + 7) / 8, sms * 8);
        router_grad_warp_kernel<<<blocks, 256, 0, st>>>(T, E, K, L.epad, bal, io.logits, io.topk_idx, io.gates, a,
                                                       io.counts, dl, dl_b);
        check(cudaGetLastError());
        const size_t n = static_cast<size_t>(E) * d;
        f32_to_bf16_kernel<<<static_cast<unsigned>(std::min<size_t>((n + 255) / 256, sms * 8)), 256, 0, st>>>(
            n, io.W_r, w_rb);
        check(cudaGetLastError());
        ex.launches += 2;
    }
    // dW_r = dl^T x: a weight gradient over the T tokens, split in token
    // chunks (partials summed in split order)
    {
        BwdGemmArgs ga;
        ga.g[0] = group0();
        ga.g[1] = group0();
        ga.status = status;
        BwdGemmGroup& r = ga.g[0];
        r.n_mats = L.rw_splits; r.fixed = L.rw_chunk; r.M = E; r.N = d;
        r.A = dl_b; r.a_rows = T; r.a_cols = L.epad; r.a_mat_stride = L.rw_chunk;
        r.B = x; r.b_mats = 1; r.b_rows = T; r.b_cols = d;
        r.out0 = L.rw_splits > 1 ? static_cast<void*>(rw_part) : static_cast<void*>(io.dW_r);
        r.ldc = d; r.c_mat_elems = static_cast<long long>(E) * d;
        check(launch_bwd_gemm(BWD_WGRAD, ga, st));
        if (L.rw_splits > 1) {
            const size_t n = static_cast<size_t>(E) * d;
            sum_splits_kernel<<<static_cast<unsigned>(std::min<size_t>((n + 255) / 256, sms * 8)), 256, 0, st>>>(
                n, L.rw_splits, rw_part, io.dW_r);
            check(cudaGetLastError());
            ++ex.launches;
        }
    }
    if (io.d_logit_bias) {
        if (dm.bias_mode == 0) {
            const int nch = (T + kChunkShared - 1) / kChunkShared;
            colsum_chunks_f32_kernel<kChunkShared><<<dim3((E + 255) / 256, std::min(nch, 65535)), 256, 0, st>>>(
                dl, E, T, part);
            check(cudaGetLastError());
            colsum_segments_kernel<kChunkShared><<<dim3((E + 31) / 32, 1), 256, 0, st>>>(part, E, nullptr, 1, T,
                                                                                     io.d_logit_bias, 1, 0);
            check(cudaGetLastError());
            ex.launches += 2;
        } else {
            ex.run(E, bwd::Fill{0.f, io.d_logit_bias});
        }
    }
    // router part of dx: dl W_r (K = N_r, zero-filled to a multiple of 64)
    {
        BwdGemmArgs ga;
        ga.g[0] = group0();
        ga.g[1] = group0();
        ga.status = status;
        BwdGemmGroup& r = ga.g[0];
        r.n_mats = 1; r.fixed = T; r.N = d; r.K = (E + 63) & ~63;
        r.A = dl_b; r.a_rows = T; r.a_cols = L.epad;
        r.B = w_rb; r.b_mats = 1; r.b_rows = E; r.b_cols = d;
        r.out0 = dxacc; r.ldc = d; r.c_rows = T;
        check(launch_bwd_gemm(BWD_DGRAD_F32, ga, st));
    }
    if (ex.err != cudaSuccess) { launches = ex.launches; return ex.err; }

    // padded routed rows, with the 16-row column partials of dy_p; db2
    {
        const dim3 grid((d + 2047) / 2048, std::min(Rp / kChunkRouted, 65535));
        pad_rows_kernel<<<grid, 256, 0, st>>>(E, K, d, io.offsets, poff, io.row_slot, io.gates, dout,
                                              static_cast<const bf*>(io.x_disp), x_p, dy_p, part);
        check(cudaGetLastError());
        colsum_segments_kernel<kChunkRouted><<<dim3((d + 31) / 32, E), 256, 0, st>>>(part, d, poff, E, 0, io.db2,
                                                                                    1, 0);
        check(cudaGetLastError());
        ex.launches += 2;
    }
    // 3. recompute: SiLU(z), SiLU'(z)
    {
        BwdGemmArgs ga;
        ga.g[0] = group0();
        ga.g[1] = group0();
        ga.status = status;
        BwdGemmGroup& r = ga.g[0];
        r.n_mats = E; r.seg = poff; r.N = dff; r.K = d;
        r.A = x_p; r.a_rows = Rp; r.a_cols = d;
        r.B = io.W1; r.b_mats = E; r.b_rows = dff; r.b_cols = d; r.b_z_mat = 1;
        r.bias = io.b1; r.out0 = h_p; r.out1 = sp_p; r.ldc = dff; r.c_rows = Rp;
        if (S > 0) {
            BwdGemmGroup& s = ga.g[1];
            s.n_mats = 1; s.fixed = T; s.N = sw; s.K = d;
            s.A = x; s.a_rows = T; s.a_cols = d;
            s.B = io.Ws1; s.b_mats = 1; s.b_rows = sw; s.b_cols = d;
            s.bias = io.bs1; s.out0 = h_s; s.out1 = sp_s; s.ldc = sw; s.c_rows = T;
        }
        check(launch_bwd_gemm(BWD_RECOMPUTE, ga, st));    // counts its own launch
    }
    // 4. dz = (dy W2) * SiLU'(z)
    {
        BwdGemmArgs ga;
        ga.g[0] = group0();
        ga.g[1] = group0();
        ga.status = status;
        BwdGemmGroup& r = ga.g[0];
        r.n_mats = E; r.seg = poff; r.N = dff; r.K = d;
        r.A = dy_p; r.a_rows = Rp; r.a_cols = d;
        r.B = io.W2; r.b_mats = E; r.b_rows = d; r.b_cols = dff; r.b_z_mat = 1;
        r.aux = sp_p; r.out0 = dz_p; r.ldc = dff; r.c_rows = Rp;
        if (S > 0) {
            BwdGemmGroup& s = ga.g[1];
            s.n_mats = S; s.fixed = T; s.N = dffs; s.K = d;
            s.A = dout; s.a_rows = T; s.a_cols = d;
            s.B = io.Ws2; s.b_mats = S; s.b_rows = d; s.b_cols = dffs; s.b_z_mat = 1;
            s.aux = sp_s; s.out0 = dz_s; s.ldc = sw; s.c_col_stride = dffs; s.c_rows = T;
        }
        check(launch_bwd_gemm(BWD_DGRAD_SILU, ga, st));
    }
    // 5. dx rows = dz W1 (routed, per padded row), dz_s Ws1 (shared, all at once)
    {
        BwdGemmArgs ga;
        ga.g[0] = group0();
        ga.g[1] = group0();
        ga.status = status;
        BwdGemmGroup& r = ga.g[0];
        r.n_mats = E; r.seg = poff; r.N = d; r.K = dff;
        r.A = dz_p; r.a_rows = Rp; r.a_cols = dff;
        r.B = io.W1; r.b_mats = E; r.b_rows = dff; r.b_cols = d; r.b_z_mat = 1;
        r.out0 = dxr_p; r.ldc = d; r.out_bf16 = 1; r.c_rows = Rp;
        if (S > 0) {
            BwdGemmGroup& s = ga.g[1];
            s.n_mats = 1; s.fixed = T; s.N = d; s.K = sw;
            s.A = dz_s; s.a_rows = T; s.a_cols = sw;
            s.B = io.Ws1; s.b_mats = 1; s.b_rows = sw; s.b_cols = d;
            s.out0 = dx_s; s.ldc = d; s.c_rows = T;
        }
        check(launch_bwd_gemm(BWD_DGRAD_F32, ga, st));
    }
    // 6a. dW2 = dy^T SiLU(z)
    {
        BwdGemmArgs ga;
        ga.g[0] = group0();
        ga.g[1] = group0();
        ga.status = status;
        BwdGemmGroup& r = ga.g[0];
        r.n_mats = E; r.seg = poff; r.M = d; r.N = dff;
        r.A = dy_p; r.a_rows = Rp; r.a_cols = d;
        r.B = h_p; r.b_mats = 1; r.b_rows = Rp; r.b_cols = dff;
        r.out0 = io.dW2; r.ldc = dff; r.c_mat_elems = static_cast<long long>(d) * dff;
        if (S > 0) {
            BwdGemmGroup& s = ga.g[1];
            s.n_mats = S; s.fixed = T; s.M = d; s.N = dffs;
            s.A = dout; s.a_rows = T; s.a_cols = d;
            s.B = h_s; s.b_mats = 1; s.b_rows = T; s.b_cols = sw; s.b_col_stride = dffs;
            s.out0 = io.dWs2; s.ldc = dffs; s.c_mat_elems = static_cast<long long>(d) * dffs;
        }
        check(launch_bwd_gemm(BWD_WGRAD, ga, st));
    }
    // 6b. dW1 = dz^T x
    {
        BwdGemmArgs ga;
        ga.g[0] = group0();
        ga.g[1] = group0();
        ga.status = status;
        BwdGemmGroup& r = ga.g[0];
        r.n_mats = E; r.seg = poff; r.M = dff; r.N = d;
        r.A = dz_p; r.a_rows = Rp; r.a_cols = dff;
        r.B = x_p; r.b_mats = 1; r.b_rows = Rp; r.b_cols = d;
        r.out0 = io.dW1; r.ldc = d; r.c_mat_elems = static_cast<long long>(dff) * d;
        if (S > 0) {
            BwdGemmGroup& s = ga.g[1];
            s.n_mats = 1; s.fixed = T; s.M = sw; s.N = d;
            s.A = dz_s; s.a_rows = T; s.a_cols = sw;
            s.B = x; s.b_mats = 1; s.b_rows = T; s.b_cols = d;
            s.out0 = io.dWs1; s.ldc = d;
        }
        check(launch_bwd_gemm(BWD_WGRAD, ga, st));
    }
    if (ex.err != cudaSuccess) { launches = ex.launches; return ex.err; }

    // 7. bias gradients
    auto colsum_routed = [&](const bf* M, int ncols, float* out) {
        const dim3 g1((ncols / 2 + 255) / 256, std::min(Rp / kChunkRouted, 65535));
        colsum_chunks_kernel<kChunkRouted><<<g1, 256, 0, st>>>(M, ncols, ncols, poff + E, 0, part);
        check(cudaGetLastError());
        colsum_segments_kernel<kChunkRouted><<<dim3((ncols + 31) / 32, E), 256, 0, st>>>(part, ncols, poff, E,
                                                                                        0, out, 1, 0);
        check(cudaGetLastError());
        ex.launches += 2;
    };
    auto colsum_shared = [&](const bf* M, int ncols, float* out, int copies, int copy_stride) {
        const dim3 g1((ncols / 2 + 255) / 256, std::min((T + kChunkShared - 1) / kChunkShared, 65535));
        colsum_chunks_kernel<kChunkShared><<<g1, 256, 0, st>>>(M, ncols, ncols, nullptr, T, part);
        check(cudaGetLastError());
        colsum_segments_kernel<kChunkShared><<<dim3((ncols + 31) / 32, 1), 256, 0, st>>>(part, ncols, nullptr, 1,
                                                                                        T, out, copies, copy_stride);
        check(cudaGetLastError());
        ex.launches += 2;
    };
    colsum_routed(dz_p, dff, io.db1);
    if (S > 0) {
        colsum_shared(dout, d, io.dbs2, S, d);
        colsum_shared(dz_s, sw, io.dbs1, 1, 0);
    }

    // 8. dx
    {
        const size_t n = static_cast<size_t>(T) * d;
        const int blocks = static_cast<int>(std::min<size_t>((n + 255) / 256, static_cast<size_t>(sms) * 16));
        dx_final_kernel<<<blocks, 256, 0, st>>>(T, K, d, dm.passthrough, dxacc, S > 0 ? dx_s : nullptr,
                                                io.slot_row, io.topk_idx, io.offsets, poff, io.gates, dxr_p,
                                                dout, io.dx);
        check(cudaGetLastError());
        ++ex.launches;
    }
    launches = ex.launches;
    return ex.err;
}

}  // namespace

size_t backward_ws_bytes(const Dims& dm) {
    return dm.dtype == MOE_BF16 ? tc_layout(dm).total : bwd::bwd_layout(dm).total;
}

cudaError_t launch_backward(const Dims& dm, float lam, const moe_backward_io& io, void* bws,
                            cudaStream_t st) {
    if (dm.dtype == MOE_BF16) {
        int launches = 0;
        const cudaError_t e = run_backward_bf16(dm, lam, io, bws, st, launches);
        count_launches(launches);
        return e;
    }
    GpuExec ex{st, cudaSuccess, 0, device_sm_count() * 16};
    bwd::run_backward(ex, dm, lam, io, bws);
    count_launches(ex.launches);
    return ex.err;
}

}  // namespace moe

// Backward of the layer: gradients of J = sum_t <dout_t, out_t> + lam * L_balance
// with respect to x, the router weight, the per-expert logit bias and every
// expert's weights and biases, for fp32 and bf16 layers.
//
// The pages define the forward only -- "論文解説: DeepSeekMoE"
// §共有エキスパート機構 (the layer output), §ルーティングとバランス損失 (s, the
// gates g_j = s_j / sum_TopK s_k, L = alpha N_r sum_j f_j P_j), §アルゴリズム
// (expert = Linear + bias -> SiLU -> Linear + bias); "Sparse MoE Top-K
// ルーティング" §解決策2 (capacity, overflow dropped or passed through).  This is
// the derivative of that forward:
//   * the top-K choice, the capacity decisions and f_j (a fraction of counts)
//     are piecewise constant and pass no gradient;
//   * slot (t, k): a = <dout_t, y_slot> if kept, <dout_t, x_t> if dropped with
//     pass-through, else 0; with S = sum_TopK s, ds_{idx_k} += (a_k -
//     sum_k' a_k' g_k') / S; P_j = mean_t s_tj adds lam alpha N_r f_j / T to
//     every ds_tj; dl = s (ds - <s, ds>); dW_r = dl^T x, dx += dl W_r, and a
//     logit bias added to the logits gets sum_t dl (a selection-only bias none);
//   * a kept slot's expert sees dy = g dout_t; shared experts dy = dout_t;
//     z = W1 x + b1, dz = (W2^T dy) * SiLU'(z), dW2 = dy SiLU(z)^T,
//     dW1 = dz x^T, db = column sums, dx = W1^T dz summed back per token;
//     a dropped slot with pass-through adds g dout_t to dx.
//
// First form of this path: every step is a functor computing one output
// element per call with a fixed-order loop over its reduction -- no atomics,
// no shared memory, bit-reproducible.  run_backward() sequences the steps
// over an executor that launches each functor as one grid-stride kernel.
#pragma once

#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include "internal.h"

namespace moe {
namespace bwd {

#define MOE_HD __host__ __device__ __forceinline__

template <typename T> MOE_HD float ld(const T* p, size_t i);
template <> MOE_HD float ld<float>(const float* p, size_t i) { return p[i]; }
template <> MOE_HD float ld<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }

MOE_HD float sigmoid_f(float z) { return 1.0f / (1.0f + expf(-z)); }
MOE_HD float silu_f(float z) { return z * sigmoid_f(z); }
MOE_HD float silu_grad_f(float z) {
    const float sg = sigmoid_f(z);
    return sg * (1.0f + z * (1.0f - sg));
}

// Rows of a step: routed rows (count offsets[N_r] on the device, expert of a
// row through row_slot and topk_idx) or the T rows of one shared expert.
struct RowMap {
    const int32_t* n_dev;       // routed: &offsets[N_r]; null for shared
    int n;                      // shared: T
    const int32_t* row_slot;    // routed: row -> t*K + k; null for shared
    const int32_t* topk_idx;
    MOE_HD int rows() const { return n_dev ? *n_dev : n; }
    MOE_HD int expert(int r) const { return row_slot ? topk_idx[row_slot[r]] : 0; }
};

// Row segment of expert e: [offsets[e], offsets[e+1]) routed, [0, n) shared.
struct Seg {
    const int32_t* offsets;
    int n;
    MOE_HD int lo(int e) const { return offsets ? offsets[e] : 0; }
    MOE_HD int hi(int e) const { return offsets ? offsets[e + 1] : n; }
};

// a[t*K + k]: dJ/dg of slot (t, k).
template <typename XT> struct GateGrad {
    int K, d, passthrough;
    const int32_t* slot_row;
    const XT *dout, *y, *x;
    float* a;
    MOE_HD void operator()(size_t i) const {
        const size_t t = i / K;
        const int row = slot_row[i];
        float acc = 0.f;
        if (row >= 0) {
            for (int c = 0; c < d; ++c) acc += ld(dout, t * d + c) * ld(y, static_cast<size_t>(row) * d + c);
        } else if (row == -1 && passthrough) {
            for (int c = 0; c < d; ++c) acc += ld(dout, t * d + c) * ld(x, t * d + c);
        }
        a[i] = acc;
    }
};

// dl[t*E + j]: dJ/dl of token t (softmax of its logits, the gates' and the
// balance loss's share of ds).
struct RouterGrad {
    int T, E, K;
    float bal;                  // lam * alpha * N_r / (T * T * K): times counts_j gives the P term
    const float* logits;        // (T, E): the logits the softmax saw
    const int32_t* topk_idx;
    const float* gates;
    const float* a;
    const int32_t* counts;
    float* dl;
    MOE_HD float ds_of(size_t t, int j, float S, float common) const {
        float v = bal * static_cast<float>(counts[j]);
        for (int k = 0; k < K; ++k)
            if (topk_idx[t * K + k] == j) v += (a[t * K + k] - common) / S;
        return v;
    }
    MOE_HD void operator()(size_t t) const {
        const float* l = logits + t * E;
        float m = l[0];
        for (int j = 1; j < E; ++j) m = fmaxf(m, l[j]);
        float z = 0.f;
        for (int j = 0; j < E; ++j) z += expf(l[j] - m);
        float S = 0.f, common = 0.f;
        for (int k = 0; k < K; ++k) {
            const int j = topk_idx[t * K + k];
            if (j >= 0 && j < E) S += expf(l[j] - m) / z;
            common += a[t * K + k] * gates[t * K + k];
        }
        float sds = 0.f;
        for (int j = 0; j < E; ++j) sds += (expf(l[j] - m) / z) * ds_of(t, j, S, common);
        for (int j = 0; j < E; ++j) {
            const float s = expf(l[j] - m) / z;
            dl[t * E + j] = s * (ds_of(t, j, S, common) - sds);
        }
    }
};

// dW_r[j*d + c] = sum_t dl[t][j] x[t][c]
template <typename XT> struct RouterWGrad {
    int T, E, d;
    const float* dl;
    const XT* x;
    float* dW_r;
    MOE_HD void operator()(size_t i) const {
        const size_t j = i / d, c = i % d;
        float acc = 0.f;
        for (int t = 0; t < T; ++t) acc += dl[static_cast<size_t>(t) * E + j] * ld(x, static_cast<size_t>(t) * d + c);
        dW_r[i] = acc;
    }
};

// out[t*d + c] = sum_j dl[t][j] W_r[j][c]
struct RouterDx {
    int E, d;
    const float* dl;
    const float* W_r;
    float* out;
    MOE_HD void operator()(size_t i) const {
        const size_t t = i / d, c = i % d;
        float acc = 0.f;
        for (int j = 0; j < E; ++j) acc += dl[t * E + j] * W_r[static_cast<size_t>(j) * d + c];
        out[i] = acc;
    }
};

// out[e*n + j] = sum over the rows r of segment e of M[r*n + j]
struct ColSum {
    Seg seg;
    int n;
    const float* M;
    float* out;
    MOE_HD void operator()(size_t i) const {
        const int e = static_cast<int>(i / n);
        const size_t j = i % n;
        float acc = 0.f;
        for (int r = seg.lo(e); r < seg.hi(e); ++r) acc += M[static_cast<size_t>(r) * n + j];
        out[i] = acc;
    }
};

struct Fill {
    float v;
    float* out;
    MOE_HD void operator()(size_t i) const { out[i] = v; }
};

// dy[r*d + c] = g of row r's slot * dout[t(r)][c], rows below offsets[N_r]
template <typename XT> struct DyRows {
    int K, d;
    const int32_t* n_dev;
    const int32_t* row_slot;
    const float* gates;
    const XT* dout;
    float* dy;
    MOE_HD void operator()(size_t i) const {
        const int r = static_cast<int>(i / d);
        if (r >= *n_dev) return;
        const size_t c = i % d;
        const int slot = row_slot[r];
        dy[i] = gates[slot] * ld(dout, static_cast<size_t>(slot / K) * d + c);
    }
};

template <typename XT> struct ToF32 {
    const XT* in;
    float* out;
    MOE_HD void operator()(size_t i) const { out[i] = ld(in, i); }
};

// z[r*f_out + f] = b1[e][f] + sum_c A[r][c] W1[e][f][c]
template <typename XT> struct ZRows {
    RowMap rm;
    int d, dff;
    const XT* A;
    const XT* W1;
    const float* b1;
    float* z;
    MOE_HD void operator()(size_t i) const {
        const int r = static_cast<int>(i / dff);
        if (r >= rm.rows()) return;
        const size_t f = i % dff;
        const size_t e = static_cast<size_t>(rm.expert(r));
        float acc = b1[e * dff + f];
        const size_t wrow = (e * dff + f) * d;
        for (int c = 0; c < d; ++c) acc += ld(A, static_cast<size_t>(r) * d + c) * ld(W1, wrow + c);
        z[i] = acc;
    }
};

// dz[r*dff + f] = (sum_c dy[r][c] W2[e][c][f]) * SiLU'(z[r][f])
template <typename XT> struct DzRows {
    RowMap rm;
    int d, dff;
    const float* dy;
    const XT* W2;
    const float* z;
    float* dz;
    MOE_HD void operator()(size_t i) const {
        const int r = static_cast<int>(i / dff);
        if (r >= rm.rows()) return;
        const size_t f = i % dff;
        const size_t e = static_cast<size_t>(rm.expert(r));
        float acc = 0.f;
        for (int c = 0; c < d; ++c)
            acc += dy[static_cast<size_t>(r) * d + c] * ld(W2, (e * d + c) * dff + f);
        dz[i] = acc * silu_grad_f(z[i]);
    }
};

// out[r*d + c] (=, or += with accumulate) sum_f dz[r][f] W1[e][f][c]
template <typename XT> struct DxRows {
    RowMap rm;
    int d, dff, accumulate;
    const float* dz;
    const XT* W1;
    float* out;
    MOE_HD void operator()(size_t i) const {
        const int r = static_cast<int>(i / d);
        if (r >= rm.rows()) return;
        const size_t c = i % d;
        const size_t e = static_cast<size_t>(rm.expert(r));
        float acc = 0.f;
        for (int f = 0; f < dff; ++f)
            acc += dz[static_cast<size_t>(r) * dff + f] * ld(W1, (e * dff + f) * d + c);
        out[i] = accumulate ? out[i] + acc : acc;
    }
};

// dW2[e][c][f] = sum over segment e of dy[r][c] SiLU(z[r][f])
struct WGrad2 {
    Seg seg;
    int d, dff;
    const float* dy;
    const float* z;
    float* dW2;
    MOE_HD void operator()(size_t i) const {
        const int e = static_cast<int>(i / (static_cast<size_t>(d) * dff));
        const size_t rem = i % (static_cast<size_t>(d) * dff);
        const size_t c = rem / dff, f = rem % dff;
        float acc = 0.f;
        for (int r = seg.lo(e); r < seg.hi(e); ++r)
            acc += dy[static_cast<size_t>(r) * d + c] * silu_f(z[static_cast<size_t>(r) * dff + f]);
        dW2[i] = acc;
    }
};

// dW1[e][f][c] = sum over segment e of dz[r][f] A[r][c]
template <typename XT> struct WGrad1 {
    Seg seg;
    int d, dff;
    const float* dz;
    const XT* A;
    float* dW1;
    MOE_HD void operator()(size_t i) const {
        const int e = static_cast<int>(i / (static_cast<size_t>(dff) * d));
        const size_t rem = i % (static_cast<size_t>(dff) * d);
        const size_t f = rem / d, c = rem % d;
        float acc = 0.f;
        for (int r = seg.lo(e); r < seg.hi(e); ++r)
            acc += dz[static_cast<size_t>(r) * dff + f] * ld(A, static_cast<size_t>(r) * d + c);
        dW1[i] = acc;
    }
};

// dx[t][c] = acc[t][c] + sum_k (kept: dxr[row][c]; dropped with
// pass-through: g * dout[t][c])
template <typename XT> struct DxFinal {
    int K, d, passthrough;
    const float* acc;
    const int32_t* slot_row;
    const float* gates;
    const float* dxr;
    const XT* dout;
    float* dx;
    MOE_HD void operator()(size_t i) const {
        const size_t t = i / d, c = i % d;
        float v = acc[i];
        for (int k = 0; k < K; ++k) {
            const int row = slot_row[t * K + k];
            if (row >= 0) v += dxr[static_cast<size_t>(row) * d + c];
            else if (row == -1 && passthrough) v += gates[t * K + k] * ld(dout, i);
        }
        dx[i] = v;
    }
};

// ------------------------------------------------------------ workspace

struct BwdLayout {
    size_t status, a, dl, dyr, zr, dzr, dxr, dys, zs, dzs, dxacc, total;
};

inline BwdLayout bwd_layout(const Dims& dm) {
    BwdLayout L{};
    size_t off = 0;
    auto take = [&](size_t floats) {
        const size_t o = off;
        off = (off + floats * 4 + 255) & ~static_cast<size_t>(255);
        return o;
    };
    const size_t T = dm.T, R = dm.r_cap;
    L.status = take(64);
    L.a = take(T * dm.K);
    L.dl = take(T * dm.E);
    L.dyr = take(R * dm.d);
    L.zr = take(R * dm.dff);
    L.dzr = take(R * dm.dff);
    L.dxr = take(R * dm.d);
    L.dys = take(dm.S > 0 ? T * dm.d : 0);
    L.zs = take(dm.S > 0 ? T * dm.dffs : 0);
    L.dzs = take(dm.S > 0 ? T * dm.dffs : 0);
    L.dxacc = take(T * dm.d);
    L.total = off;
    return L;
}

// ------------------------------------------------------------ sequence

template <typename XT, class Exec>
void run_backward_t(Exec& ex, const Dims& dm, float lam, const moe_backward_io& io, void* bws) {
    const BwdLayout L = bwd_layout(dm);
    auto F = [&](size_t off) { return reinterpret_cast<float*>(static_cast<uint8_t*>(bws) + off); };
    float *a = F(L.a), *dl = F(L.dl), *dyr = F(L.dyr), *zr = F(L.zr), *dzr = F(L.dzr), *dxr = F(L.dxr);
    float *dys = F(L.dys), *zs = F(L.zs), *dzs = F(L.dzs), *dxacc = F(L.dxacc);
    const size_t T = dm.T, d = dm.d, E = dm.E, K = dm.K, dff = dm.dff, R = dm.r_cap;
    const XT* x = static_cast<const XT*>(io.x);
    const XT* dout = static_cast<const XT*>(io.dout);
    const XT* xd = static_cast<const XT*>(io.x_disp);

    ex.run(1, Fill{0.f, F(L.status)});                     // device status word: no waits here
    ex.run(T * K, GateGrad<XT>{dm.K, dm.d, dm.passthrough, io.slot_row, dout, static_cast<const XT*>(io.y), x, a});
    const float bal = lam * dm.alpha * static_cast<float>(dm.E) /
                      (static_cast<float>(dm.T) * static_cast<float>(dm.T) * static_cast<float>(dm.K));
    ex.run(T, RouterGrad{dm.T, dm.E, dm.K, bal, io.logits, io.topk_idx, io.gates, a, io.counts, dl});
    ex.run(E * d, RouterWGrad<XT>{dm.T, dm.E, dm.d, dl, x, io.dW_r});
    if (io.d_logit_bias) {
        if (dm.bias_mode == 0) ex.run(E, ColSum{Seg{nullptr, dm.T}, dm.E, dl, io.d_logit_bias});
        else ex.run(E, Fill{0.f, io.d_logit_bias});
    }
    ex.run(T * d, RouterDx{dm.E, dm.d, dl, io.W_r, dxacc});

    // routed experts over the dispatched rows
    const RowMap rr{io.offsets + dm.E, 0, io.row_slot, io.topk_idx};
    const Seg sr{io.offsets, 0};
    const XT* W1 = static_cast<const XT*>(io.W1);
    const XT* W2 = static_cast<const XT*>(io.W2);
    ex.run(R * d, DyRows<XT>{dm.K, dm.d, io.offsets + dm.E, io.row_slot, io.gates, dout, dyr});
    ex.run(R * dff, ZRows<XT>{rr, dm.d, dm.dff, xd, W1, io.b1, zr});
    ex.run(R * dff, DzRows<XT>{rr, dm.d, dm.dff, dyr, W2, zr, dzr});
    ex.run(E * d * dff, WGrad2{sr, dm.d, dm.dff, dyr, zr, io.dW2});
    ex.run(E * d, ColSum{sr, dm.d, dyr, io.db2});
    ex.run(E * dff * d, WGrad1<XT>{sr, dm.d, dm.dff, dzr, xd, io.dW1});
    ex.run(E * dff, ColSum{sr, dm.dff, dzr, io.db1});
    ex.run(R * d, DxRows<XT>{rr, dm.d, dm.dff, 0, dzr, W1, dxr});

    // shared experts over all T tokens, dy = dout
    if (dm.S > 0) {
        const size_t dfs = dm.dffs;
        const RowMap rs{nullptr, dm.T, nullptr, nullptr};
        const Seg ss{nullptr, dm.T};
        ex.run(T * d, ToF32<XT>{dout, dys});
        for (int s = 0; s < dm.S; ++s) {
            const XT* Ws1 = static_cast<const XT*>(io.Ws1) + static_cast<size_t>(s) * dfs * d;
            const XT* Ws2 = static_cast<const XT*>(io.Ws2) + static_cast<size_t>(s) * d * dfs;
            ex.run(T * dfs, ZRows<XT>{rs, dm.d, dm.dffs, x, Ws1, io.bs1 + s * dfs, zs});
            ex.run(T * dfs, DzRows<XT>{rs, dm.d, dm.dffs, dys, Ws2, zs, dzs});
            ex.run(d * dfs, WGrad2{ss, dm.d, dm.dffs, dys, zs, io.dWs2 + s * d * dfs});
            ex.run(d, ColSum{ss, dm.d, dys, io.dbs2 + s * d});
            ex.run(dfs * d, WGrad1<XT>{ss, dm.d, dm.dffs, dzs, x, io.dWs1 + s * dfs * d});
            ex.run(dfs, ColSum{ss, dm.dffs, dzs, io.dbs1 + s * dfs});
            ex.run(T * d, DxRows<XT>{rs, dm.d, dm.dffs, 1, dzs, Ws1, dxacc});
        }
    }
    ex.run(T * d, DxFinal<XT>{dm.K, dm.d, dm.passthrough, dxacc, io.slot_row, io.gates, dxr, dout, io.dx});
}

template <class Exec>
void run_backward(Exec& ex, const Dims& dm, float lam, const moe_backward_io& io, void* bws) {
    if (dm.dtype == MOE_F32) run_backward_t<float>(ex, dm, lam, io, bws);
    else run_backward_t<__nv_bfloat16>(ex, dm, lam, io, bws);
}

#undef MOE_HD

}  // namespace bwd
}  // namespace moe

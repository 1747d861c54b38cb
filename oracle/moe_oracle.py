"""fp64 CPU oracle of the sparse MoE FFN layer: the forward, and its backward
for the fp32 and bf16 workloads.

TEST INFRASTRUCTURE.  Only tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the CUDA
library and imports nothing from it.

Sources (reference pages, cited by page title and section):
  [DSMoE]  "論文解説: DeepSeekMoE — 細粒度エキスパート分割と共有エキスパートによる
           MoE効率化" (0h-n0.github.io): §共有エキスパート機構 (layer output h_t),
           §ルーティングとバランス損失 (gate g_j, softmax s_j, balance loss),
           §アルゴリズム (the reference nn.Module: router Linear without bias,
           expert = Linear -> SiLU -> Linear with biases, top-K, renormalise),
           §実装のポイント (alpha = 0.01).
  [TopK]   "Sparse MoE Top-Kルーティング" (jisaku.com glossary):
           §ルーティングの仕組み (top-K, gate weights, weighted sum),
           §解決策2 エキスパートキャパシティファクター and FAQ Q2 (capacity,
           overflow tokens dropped).
  [EP]     "エキスパート並列（Expert Parallelism）" (jisaku.com glossary):
           §推論フロー (route tokens to their expert and back).
  [DeepEP] "DeepSeek DeepEP" (blogs.novita.ai): §DeepEP とは item 5 and
           §DeepEP の性能 (FP8 dispatch, BF16 combine).

Readings where the pages leave a step open (each is also listed in the design
notes of the repository):
  * selection uses the logits (softmax is monotone); ties go to the lower
    expert index; slot order is descending logit, then ascending index;
  * capacity C = ceil(cf * T * K / N_r); within an expert, slots keep token
    order and the first C are kept (earliest token first); a dropped slot adds
    nothing and the other gates are not renormalised;
  * f_j uses pre-drop counts over T*K slots; P_j is the mean of the full
    softmax (including any logit bias) over all T tokens;
  * FP8: activations are quantised per row per 128 columns and weights per
    128x128 block, each with the smallest power-of-two scale 2^k such that
    amax / 2^k <= 448 (scale 1 for an all-zero block), codes by
    round-to-nearest-even with saturation to +-448; the hidden activation h is
    re-quantised the same way before the second linear layer, expert outputs
    are rounded to bf16 before the combine and the layer output is rounded to
    bf16 at the end.  In bf16 and fp32 workloads nothing is rounded in between.

Parity pins (tests/test_oracle_pins.py): gates sum to one; counts sum to T*K;
the dispatch permutation is a bijection with rows in token order; N_r = K = 1
reduces to a dense FFN checked against torch's CPU linear/SiLU; the
dense masked form of the reference module (every expert on every token, then
masked) gives the same output; brute-force top-K over all K-subsets on tiny
inputs; the C(8,2) = 28 and C(16,2) = 120 selected-set counts; active-parameter
fraction K/N_r; balance loss closed forms (uniform routing gives alpha, a
collapsed router gives alpha * N_r); the first C tokens kept under capacity;
hand-computed capacities (including fp32 values of the capacity factor);
the e4m3 and bf16 rounding against torch's conversions.  The expert FFN
arithmetic beyond these is pinned only through the dense limit.

The backward (layer_backward) is the derivative of this forward; the pages
give no backward.  Its readings: the top-K choice, the capacity decisions and
f_j are piecewise constant (no gradient through them); P_j carries the
balance-loss gradient to s; a selection-only bias gets none.  Pins
(tests/test_oracle_backward_pins.py): central differences of the forward's
objective <dout, out> + lam * L_balance over every input and weight of tiny
layers (capacity drops, pass-through, shared experts, both bias modes,
K = 1, K = N_r); closed forms for K = 1, for the balance loss alone and for
K = N_r (gates equal to the softmax).
"""
from __future__ import annotations

import math
from fractions import Fraction
from typing import Dict, Optional

import numpy as np

__all__ = [
    "E4M3_MAX", "e4m3_decode", "e4m3_round", "pow2_scale", "quantize_rows_1x128",
    "dequant_rows_1x128", "dequant_blocks_128x128", "bf16_round",
    "router_logits", "softmax", "topk_select", "gates_of", "capacity_of",
    "dispatch_plan", "silu", "expert_ffn", "balance_stats", "topk_gap",
    "route", "layer_forward", "to_f64", "expert_weights",
    "silu_grad", "expert_ffn_backward", "layer_backward", "layer_backward_sample",
]

E4M3_MAX = 448.0
_QBLOCK = 128


# ----------------------------------------------------------------------------
# Number formats ([DeepEP] FP8 dispatch / BF16 combine; format definitions:
# e4m3 = 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals,
# no infinities, S.1111.111 is NaN; bf16 = the upper half of an IEEE fp32)
# ----------------------------------------------------------------------------

def _e4m3_value(c: int) -> float:
    """Value of one e4m3 code from the format definition."""
    sign = -1.0 if c & 0x80 else 1.0
    e = (c >> 3) & 0xF
    m = c & 0x7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 e4m3 codes -> fp64 values (NaN for S.1111.111)."""
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


_E4M3_POS = e4m3_decode(np.arange(127, dtype=np.uint8))   # codes 0x00..0x7E, ascending


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Round fp64 values to e4m3 codes: nearest representable value, ties to
    the even code, magnitudes beyond 448 saturate to 448; as in IEEE
    rounding, a negative value that rounds to zero gives negative zero."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.searchsorted(_E4M3_POS, a, side="left")          # first table value >= a
    hi = np.minimum(hi, len(_E4M3_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_hi = _E4M3_POS[hi] - a
    d_lo = a - _E4M3_POS[lo]
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    # the sign is kept, also when the magnitude rounds to zero (-0 is S=1, E=0, M=0)
    code = np.where(np.signbit(v), code | 0x80, code)
    return code.astype(np.uint8)


def pow2_scale(amax: np.ndarray) -> np.ndarray:
    """Smallest power of two 2^k with amax / 2^k <= 448; 1 where amax == 0.

    Scales are stored as fp32, so k is kept in the normal fp32 exponent range
    [-126, 127] (a reading: the pages give no scale rule at all).  Only a
    block whose amax is below 448 * 2^-126 (about 5.3e-36) meets the lower
    bound; its scale is 2^-126 and its codes are then smaller than 448.  The
    upper bound is out of reach of fp32 inputs."""
    amax = np.asarray(amax, dtype=np.float64)
    out = np.ones_like(amax)
    nz = amax > 0
    k = np.ceil(np.log2(amax[nz] / E4M3_MAX))
    s = np.exp2(k)
    # guard the float log2 against an off-by-one at exact powers of two
    s = np.where(amax[nz] / s > E4M3_MAX, s * 2.0, s)
    s = np.where(amax[nz] / (s / 2.0) <= E4M3_MAX, s / 2.0, s)
    out[nz] = np.clip(s, 2.0 ** -126, 2.0 ** 127)
    return out


def quantize_rows_1x128(v: np.ndarray):
    """(rows, cols) fp64 -> e4m3 codes (rows, cols) and fp64 scales
    (rows, cols/128): one scale per row per 128 columns."""
    rows, cols = v.shape
    assert cols % _QBLOCK == 0
    vb = v.reshape(rows, cols // _QBLOCK, _QBLOCK)
    scale = pow2_scale(np.abs(vb).max(axis=2))
    codes = e4m3_round(vb / scale[:, :, None])     # division by 2^k is exact
    return codes.reshape(rows, cols), scale


def dequant_rows_1x128(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    rows, cols = codes.shape
    vals = e4m3_decode(codes).reshape(rows, cols // _QBLOCK, _QBLOCK)
    return (vals * np.asarray(scales, np.float64)[:, :, None]).reshape(rows, cols)


def dequant_blocks_128x128(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    rows, cols = codes.shape
    vals = e4m3_decode(codes).reshape(rows // _QBLOCK, _QBLOCK, cols // _QBLOCK, _QBLOCK)
    return (vals * np.asarray(scales, np.float64)[:, None, :, None]).reshape(rows, cols)


def bf16_round(v: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), returned as
    fp64.  bf16 keeps 8 significant bits; below 2^-126 the spacing is 2^-133."""
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)                      # v = m * 2^e, |m| in [0.5, 1)
    quantum = np.exp2(np.maximum(e - 8, -133).astype(np.float64))
    return np.rint(v / quantum) * quantum   # rint rounds halves to even


def to_f64(a) -> np.ndarray:
    """torch tensor / numpy array of fp32, bf16 or fp64 values -> fp64 numpy."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------
# Router ([DSMoE] §ルーティングとバランス損失: s_j = softmax(W_r x)_j,
# g_j = s_j / sum_{k in TopK} s_k; [TopK] §ルーティングの仕組み)
# ----------------------------------------------------------------------------

def router_logits(x: np.ndarray, W_r: np.ndarray, logit_bias: Optional[np.ndarray] = None) -> np.ndarray:
    """l[t, j] = sum_i x[t, i] W_r[j, i] (+ b_j), fp64.  The router is a linear
    map without bias ([DSMoE] §アルゴリズム); b_j is the decode workload's
    per-expert logit bias."""
    l = np.asarray(x, np.float64) @ np.asarray(W_r, np.float64).T
    if logit_bias is not None:
        l = l + np.asarray(logit_bias, np.float64)[None, :]
    return l


def softmax(l: np.ndarray) -> np.ndarray:
    """Softmax over all routed experts of each token."""
    z = l - l.max(axis=1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=1, keepdims=True)


def topk_select(l: np.ndarray, K: int) -> np.ndarray:
    """Indices of the K largest logits per token, in slot order: descending
    logit, equal logits by ascending expert index (the lower index wins a tie).
    A stable sort of -l keeps equal keys in index order."""
    order = np.argsort(-np.asarray(l, np.float64), axis=1, kind="stable")
    return order[:, :K].astype(np.int32)


def gates_of(s: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """g[t, k] = s[t, idx[t, k]] / sum_k' s[t, idx[t, k']]."""
    sel = np.take_along_axis(s, idx.astype(np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def topk_gap(l: np.ndarray, K: int) -> np.ndarray:
    """l_(K) - l_(K+1) of each token's descending logits (inf when K = N_r)."""
    srt = -np.sort(-np.asarray(l, np.float64), axis=1)
    if K >= srt.shape[1]:
        return np.full(srt.shape[0], np.inf)
    return srt[:, K - 1] - srt[:, K]


# ----------------------------------------------------------------------------
# Dispatch plan ([EP] §推論フロー: tokens go to the expert that serves them;
# [TopK] §解決策2 / FAQ Q2: per-expert capacity per batch, overflow dropped)
# ----------------------------------------------------------------------------

def capacity_of(T: int, K: int, N_r: int, cf: float) -> Optional[int]:
    """C = ceil(cf * T * K / N_r), evaluated exactly on the fp32 value of cf;
    None when cf <= 0 (no limit)."""
    cf32 = float(np.float32(cf))
    if cf32 <= 0:
        return None
    return int(math.ceil(Fraction(cf32) * T * K / N_r))


def dispatch_plan(idx: np.ndarray, N_r: int, C: Optional[int], priority: str = "token") -> Dict[str, np.ndarray]:
    """Counts, kept counts, segment offsets and the slot<->row permutation.

    Slots (t, k) of expert j are ranked in ascending token order
    (priority "token", [TopK] FAQ Q2: the earliest tokens are kept), or
    slot-major (priority "slot": every token's k-th choice before any
    (k+1)-th choice, each in token order); slot of rank r is kept iff r < C.
    Kept slots of expert j occupy rows offsets[j] .. offsets[j] + kept[j] - 1
    in rank order.
    """
    T, K = idx.shape
    counts = np.zeros(N_r, np.int64)
    rank = np.full((T, K), -1, np.int64)
    order = ([(t, k) for t in range(T) for k in range(K)] if priority == "token"
             else [(t, k) for k in range(K) for t in range(T)])
    for t, k in order:
        j = int(idx[t, k])
        rank[t, k] = counts[j]
        counts[j] += 1
    kept = counts.copy() if C is None else np.minimum(counts, C)
    offsets = np.zeros(N_r + 1, np.int64)
    offsets[1:] = np.cumsum(kept)
    R = int(offsets[-1])
    slot_row = np.full((T, K), -1, np.int64)
    row_slot = np.full(R, -1, np.int64)
    for t in range(T):
        for k in range(K):
            j = int(idx[t, k])
            if C is None or rank[t, k] < C:
                r = int(offsets[j] + rank[t, k])
                slot_row[t, k] = r
                row_slot[r] = t * K + k
    return {"counts": counts, "kept": kept, "offsets": offsets,
            "slot_row": slot_row, "row_slot": row_slot, "R": R}


# ----------------------------------------------------------------------------
# Expert FFN ([DSMoE] §アルゴリズム: Linear(d, d_ff) + bias -> SiLU ->
# Linear(d_ff, d) + bias)
# ----------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def expert_ffn(xr: np.ndarray, W1: np.ndarray, b1: np.ndarray, W2: np.ndarray,
               b2: np.ndarray, fp8_hidden: bool = False) -> np.ndarray:
    """y = W2 SiLU(W1 x + b1) + b2 for each row of xr, fp64.  With fp8_hidden
    the hidden activation is quantised per row per 128 columns first."""
    h = silu(xr @ W1.T + b1[None, :])
    if fp8_hidden:
        codes, sc = quantize_rows_1x128(h)
        h = dequant_rows_1x128(codes, sc)
    return h @ W2.T + b2[None, :]


# ----------------------------------------------------------------------------
# Balance statistics ([DSMoE] §ルーティングとバランス損失:
# L = alpha * N_r * sum_j f_j P_j)
# ----------------------------------------------------------------------------

def balance_stats(counts: np.ndarray, s: np.ndarray, K: int, alpha: float):
    T, N_r = s.shape
    f = np.asarray(counts, np.float64) / float(T * K)
    P = s.mean(axis=0)
    L = alpha * N_r * float(np.sum(f * P))
    return f, P, L


# ----------------------------------------------------------------------------
# Whole layer ([DSMoE] §共有エキスパート機構: h_t = sum_i E_s,i(x_t)
# + sum_{j in TopK} g_j(x_t) E_r,j(x_t))
# ----------------------------------------------------------------------------

def route(shape, inputs, logits: Optional[np.ndarray] = None):
    """Router, top-K, gates, plan and balance statistics for all T tokens.

    A per-expert bias b is used in one of two ways (shape.bias_mode):
      0  added to the logits: s, top-K, gates and P all see l + b (the decode
         workload's skew);
      1  selection only ([TopK] §解決策3, auxiliary-loss-free balancing: a
         per-expert bias steers which experts are chosen, the loss is not
         changed): top-K on l + b, while s, the gates and P use the unbiased
         l.  The pages give no formula; this is the plainest reading.

    `logits`, when given, replaces the oracle's own fp64 logits as the
    selection keys (used to check the product's routing bit-exactly on its own
    fp32 logits -- those are l + b in mode 0 and l in mode 1, to which the
    bias is then added in fp32 as the kernel does); s and P still come from
    the oracle's fp64 logits."""
    x = to_f64(inputs["x"])
    lb = inputs.get("logit_bias")
    mode = getattr(shape, "bias_mode", 0)
    sel_bias = None if (lb is None or mode != 1) else to_f64(lb)
    l64 = router_logits(x, to_f64(inputs["W_r"]), None if (lb is None or mode == 1) else to_f64(lb))
    s = softmax(l64)
    keys64 = l64 if sel_bias is None else l64 + sel_bias[None, :]
    if logits is None:
        keys = keys64
    elif sel_bias is None:
        keys = np.asarray(logits, np.float64)
    else:
        b32 = np.asarray(to_f64(lb), np.float32)
        keys = (np.asarray(logits, np.float32) + b32[None, :]).astype(np.float64)
    idx = topk_select(keys, shape.top_k)
    g = gates_of(s, idx)
    C = capacity_of(shape.T, shape.top_k, shape.n_routed, shape.capacity_factor)
    plan = dispatch_plan(idx, shape.n_routed, C,
                         "slot" if getattr(shape, "capacity_priority", 0) == 1 else "token")
    f, P, L = balance_stats(plan["counts"], s, shape.top_k, shape.alpha)
    return {"logits": l64, "s": s, "idx": idx, "gates": g, "C": C, "plan": plan,
            "f": f, "P": P, "loss": L, "gap": topk_gap(keys64, shape.top_k)}


def expert_weights(inputs, prefix: str, e: int, fp8: bool):
    """fp64 (W1, b1, W2, b2) of routed (prefix 'W') or shared (prefix 'Ws')
    expert e."""
    b = "b" if prefix == "W" else "bs"
    if fp8:
        W1 = dequant_blocks_128x128(_np_u8(inputs[prefix + "1"][e]), to_f64(inputs[prefix + "1_scales"][e]))
        W2 = dequant_blocks_128x128(_np_u8(inputs[prefix + "2"][e]), to_f64(inputs[prefix + "2_scales"][e]))
    else:
        W1 = to_f64(inputs[prefix + "1"][e])
        W2 = to_f64(inputs[prefix + "2"][e])
    return W1, to_f64(inputs[b + "1"][e]), W2, to_f64(inputs[b + "2"][e])


def _np_u8(a) -> np.ndarray:
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu").view(torch.uint8).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, np.uint8)


def layer_forward(shape, inputs, tokens: Optional[np.ndarray] = None,
                  routing: Optional[dict] = None) -> dict:
    """The layer output for `tokens` (default: all T), plus the routing.

    Returns {"out": (len(tokens), d) fp64, "tokens", "routing"}.  Each token's
    output is sum_k g[t, k] * E_{idx[t, k]}(x_t) over its kept slots in
    ascending k, then the shared experts in ascending order.  In FP8 workloads
    x is quantised per row per 128 columns before the experts, h is
    re-quantised, each expert output is rounded to bf16 and the sum is rounded
    to bf16 at the end.
    """
    fp8 = shape.dtype == 2
    rt = routing if routing is not None else route(shape, inputs)
    T, K = shape.T, shape.top_k
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, np.int64)
    x = to_f64(inputs["x"])[tokens]
    if fp8:
        xc, xs = quantize_rows_1x128(x)
        xin = dequant_rows_1x128(xc, xs)
    else:
        xin = x
    slot_row = rt["plan"]["slot_row"]
    # expert outputs of every kept slot of the requested tokens, one expert at a time
    by_expert: Dict[int, list] = {}
    for i, t in enumerate(tokens):
        for k in range(K):
            if slot_row[t, k] >= 0:
                by_expert.setdefault(int(rt["idx"][t, k]), []).append((i, k))
    y_slot: Dict[tuple, np.ndarray] = {}
    for e in sorted(by_expert):
        W1, b1, W2, b2 = expert_weights(inputs, "W", e, fp8)
        rows = by_expert[e]
        y = expert_ffn(xin[np.array([i for i, _ in rows])], W1, b1, W2, b2, fp8_hidden=fp8)
        if fp8:
            y = bf16_round(y)
        for n, key in enumerate(rows):
            y_slot[key] = y[n]
    out = np.zeros((len(tokens), shape.d_model), np.float64)
    # [TopK] §解決策2: a slot over the capacity is dropped, or (overflow_mode 1)
    # the token passes that expert unchanged: its own input times its gate
    passthrough = getattr(shape, "overflow_mode", 0) == 1
    for i, t in enumerate(tokens):
        for k in range(K):
            if (i, k) in y_slot:
                out[i] += rt["gates"][t, k] * y_slot[(i, k)]
            elif passthrough:
                out[i] += rt["gates"][t, k] * x[i]
    for s_i in range(shape.n_shared):
        W1, b1, W2, b2 = expert_weights(inputs, "Ws", s_i, fp8)
        y = expert_ffn(xin, W1, b1, W2, b2, fp8_hidden=fp8)
        if fp8:
            y = bf16_round(y)
        out += y
    if fp8:
        out = bf16_round(out)
    return {"out": out, "tokens": tokens, "routing": rt}


# ----------------------------------------------------------------------------
# Backward of the layer (the derivative of what the forward above computes;
# the pages state the forward only: [DSMoE] §共有エキスパート機構 for the
# output, §ルーティングとバランス損失 for the gates and the balance loss,
# §アルゴリズム for the expert module; [TopK] §解決策2 for the capacity and the
# overflow pass-through)
# ----------------------------------------------------------------------------

def silu_grad(z: np.ndarray) -> np.ndarray:
    """d SiLU / dz = sigma(z) (1 + z (1 - sigma(z)))."""
    sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


def expert_ffn_backward(xr: np.ndarray, dy: np.ndarray, W1: np.ndarray, b1: np.ndarray,
                        W2: np.ndarray) -> dict:
    """Gradients of y = W2 SiLU(W1 x + b1) + b2 over the rows of xr, given
    dy = dJ/dy per row: dx (rows, d), dW1, db1, dW2, db2 summed over rows."""
    z = xr @ W1.T + b1[None, :]
    h = silu(z)
    dh = dy @ W2
    dz = dh * silu_grad(z)
    return {"dx": dz @ W1, "dW1": dz.T @ xr, "db1": dz.sum(axis=0),
            "dW2": dy.T @ h, "db2": dy.sum(axis=0)}


def layer_backward(shape, inputs, dout: np.ndarray, lam: float = 1.0,
                   routing: Optional[dict] = None) -> dict:
    """Gradients of J = sum_t <dout_t, out_t> + lam * L_balance with respect
    to x, the router weight, the per-expert bias and every expert's weights,
    for the fp32 and bf16 workloads (fp64 throughout, nothing rounded).

    Readings (the pages give no backward; this is the derivative of the
    forward as the oracle computes it):
      * the top-K choice, the capacity decisions and f_j (a fraction of
        counts) are piecewise constant: no gradient flows through them;
      * with S = sum_{k in TopK} s_k and g_k = s_{idx_k} / S, a slot's gate
        gradient a_k = <dout_t, y_k> (kept), <dout_t, x_t> (dropped with
        pass-through) or 0 (dropped), and ds_{idx_m} = (a_m - sum_k a_k g_k) / S;
      * P_j = mean_t s_tj adds lam * alpha * N_r * f_j / T to every ds_tj;
      * softmax: dl_i = s_i (ds_i - sum_j s_j ds_j); the router is linear, so
        dW_r = dl^T x, dx += dl W_r, and the bias gets sum_t dl when it is
        added to the logits (bias_mode 0); a selection-only bias (bias_mode 1)
        enters only the top-K keys and gets none;
      * a kept slot's expert sees dy = g_k dout_t; a dropped slot with
        pass-through adds g_k dout_t to dx; shared experts see dy = dout_t.

    Returns a dict with "x" (T, d), "W_r" (N_r, d), "logit_bias" (N_r,) or
    None, "W1", "b1", "W2", "b2" (stacked over routed experts), "Ws1", "bs1",
    "Ws2", "bs2" (shared, or None) and the intermediates "dgates" (T, K),
    "ds" (T, N_r) and "dlogits" (T, N_r).
    """
    if shape.dtype == 2:
        raise ValueError("layer_backward covers the fp32 and bf16 workloads")
    rt = routing if routing is not None else route(shape, inputs)
    T, K, N_r = shape.T, shape.top_k, shape.n_routed
    x = to_f64(inputs["x"])
    dout = np.asarray(dout, np.float64)
    W_r = to_f64(inputs["W_r"])
    s, idx, g = rt["s"], rt["idx"].astype(np.int64), rt["gates"]
    slot_row = rt["plan"]["slot_row"]
    passthrough = getattr(shape, "overflow_mode", 0) == 1
    dx = np.zeros_like(x)
    d_exp = {k: [] for k in ("W1", "b1", "W2", "b2")}
    a = np.zeros((T, K), np.float64)                 # dJ/dg per slot
    for e in range(N_r):
        W1, b1, W2, b2 = expert_weights(inputs, "W", e, False)
        slots = [(t, k) for t in range(T) for k in range(K) if idx[t, k] == e and slot_row[t, k] >= 0]
        if slots:
            tt = np.array([t for t, _ in slots])
            kk = np.array([k for _, k in slots])
            xr = x[tt]
            y = expert_ffn(xr, W1, b1, W2, b2)
            a[tt, kk] = np.einsum("rd,rd->r", dout[tt], y)
            gb = expert_ffn_backward(xr, g[tt, kk][:, None] * dout[tt], W1, b1, W2)
            np.add.at(dx, tt, gb["dx"])
        else:
            gb = {"dW1": np.zeros_like(W1), "db1": np.zeros_like(b1),
                  "dW2": np.zeros_like(W2), "db2": np.zeros_like(b2)}
        for k in d_exp:
            d_exp[k].append(gb["d" + k])
    for t in range(T):
        for k in range(K):
            if slot_row[t, k] < 0 and passthrough:
                a[t, k] = float(dout[t] @ x[t])
                dx[t] += g[t, k] * dout[t]
    # gates -> s over the selected experts of each token
    S = np.take_along_axis(s, idx, axis=1).sum(axis=1)
    ds = np.zeros_like(s)
    common = (a * g).sum(axis=1)
    for t in range(T):
        for k in range(K):
            ds[t, idx[t, k]] += (a[t, k] - common[t]) / S[t]
    # balance loss through P (f held constant)
    f = rt["f"]
    ds += lam * shape.alpha * N_r * f[None, :] / T
    # softmax and the linear router
    dl = s * (ds - (s * ds).sum(axis=1, keepdims=True))
    dx += dl @ W_r
    lb = inputs.get("logit_bias")
    d_bias = None
    if lb is not None:
        d_bias = dl.sum(axis=0) if getattr(shape, "bias_mode", 0) == 0 else np.zeros(N_r)
    shared = {k: None for k in ("Ws1", "bs1", "Ws2", "bs2")}
    if shape.n_shared > 0:
        parts = {k: [] for k in shared}
        for si in range(shape.n_shared):
            W1, b1, W2, b2 = expert_weights(inputs, "Ws", si, False)
            gb = expert_ffn_backward(x, dout, W1, b1, W2)
            dx += gb["dx"]
            for k in ("W1", "b1", "W2", "b2"):
                parts[("Ws" if k[0] == "W" else "bs") + k[1]].append(gb["d" + k])
        shared = {k: np.stack(v) for k, v in parts.items()}
    res = {"x": dx, "W_r": dl.T @ x, "logit_bias": d_bias,
           "dgates": a, "ds": ds, "dlogits": dl}
    for k in d_exp:
        res[k] = np.stack(d_exp[k])
    res.update(shared)
    return res


def layer_backward_sample(shape, inputs, dout: np.ndarray, lam: float, routing: dict,
                          experts, f_idx, c_idx, tokens, fs_idx=None) -> dict:
    """Selected entries of layer_backward, each computed from the same
    definitions with only the work it needs, so that layers of full size can
    be checked:
      "W1"[e]  dW1[e][f_idx, :]         "b1"[e]  db1[e][f_idx]
      "W2"[e]  dW2[e][c_idx][:, f_idx]  "b2"[e]  db2[e][c_idx]
    for each routed expert e in `experts`,
      "Ws1"[s] dWs1[s][fs_idx, :]       "bs1"[s] dbs1[s][fs_idx]
      "Ws2"[s] dWs2[s][c_idx][:, fs_idx] "bs2"[s] dbs2[s][c_idx]
    for every shared expert s, and "x" = dx[tokens].  routing: the output of
    route() for the whole batch (the balance term needs f over all tokens).
    The derivative read is layer_backward's: a kept slot's expert sees
    dy = g dout_t; a token's dx is its router part dl_t W_r, its kept slots'
    W1^T dz, g dout_t for slots passed through and its shared experts'."""
    if shape.dtype == 2:
        raise ValueError("layer_backward_sample covers the fp32 and bf16 workloads")
    rt = routing
    T, K, N_r = shape.T, shape.top_k, shape.n_routed
    f_idx, c_idx = np.asarray(f_idx), np.asarray(c_idx)
    fs_idx = f_idx if fs_idx is None else np.asarray(fs_idx)
    s, idx, g = rt["s"], rt["idx"].astype(np.int64), rt["gates"]
    slot_row = rt["plan"]["slot_row"]
    passthrough = getattr(shape, "overflow_mode", 0) == 1

    def xrow(ts):
        return to_f64(inputs["x"][np.asarray(ts)]) if len(ts) else np.zeros((0, shape.d_model))

    def drow(ts):
        return np.asarray(dout, np.float64)[np.asarray(ts)]

    res = {k: {} for k in ("W1", "b1", "W2", "b2", "Ws1", "bs1", "Ws2", "bs2")}
    for e in experts:
        W1, b1, W2, b2 = expert_weights(inputs, "W", e, False)
        slots = [(t, k) for t in range(T) for k in range(K) if idx[t, k] == e and slot_row[t, k] >= 0]
        tt = [t for t, _ in slots]
        xr = xrow(tt)
        dy = np.array([g[t, k] for t, k in slots])[:, None] * drow(tt) if slots else np.zeros((0, shape.d_model))
        z = xr @ W1[f_idx].T + b1[f_idx][None, :]
        dz = (dy @ W2[:, f_idx]) * silu_grad(z)
        res["W1"][e] = dz.T @ xr
        res["b1"][e] = dz.sum(axis=0)
        res["W2"][e] = dy[:, c_idx].T @ silu(z)
        res["b2"][e] = dy[:, c_idx].sum(axis=0)
    if shape.n_shared > 0:
        xa = to_f64(inputs["x"])
        da = np.asarray(dout, np.float64)
        for si in range(shape.n_shared):
            W1, b1, W2, b2 = expert_weights(inputs, "Ws", si, False)
            z = xa @ W1[fs_idx].T + b1[fs_idx][None, :]
            dz = (da @ W2[:, fs_idx]) * silu_grad(z)
            res["Ws1"][si] = dz.T @ xa
            res["bs1"][si] = dz.sum(axis=0)
            res["Ws2"][si] = da[:, c_idx].T @ silu(z)
            res["bs2"][si] = da[:, c_idx].sum(axis=0)
    # dx of the chosen tokens: each expert's weights are widened once for all
    # the chosen tokens' slots it serves
    W_r = to_f64(inputs["W_r"])
    f = rt["f"]
    tokens = [int(t) for t in tokens]
    xt_all = {t: to_f64(inputs["x"][t]) for t in tokens}
    dt_all = {t: np.asarray(dout[t], np.float64) for t in tokens}
    a = {t: np.zeros(K) for t in tokens}
    v = {t: np.zeros(shape.d_model) for t in tokens}
    by_expert = {}
    for t in tokens:
        for k in range(K):
            if slot_row[t, k] >= 0:
                by_expert.setdefault(int(idx[t, k]), []).append((t, k))
            elif passthrough:
                a[t][k] = float(dt_all[t] @ xt_all[t])
                v[t] += g[t, k] * dt_all[t]
    for e, slots_e in by_expert.items():
        W1, b1, W2, b2 = expert_weights(inputs, "W", e, False)
        for t, k in slots_e:
            xt, dt = xt_all[t], dt_all[t]
            a[t][k] = float(dt @ expert_ffn(xt[None, :], W1, b1, W2, b2)[0])
            z = W1 @ xt + b1
            v[t] += ((W2.T @ (g[t, k] * dt)) * silu_grad(z)) @ W1
    for si in range(shape.n_shared):
        W1, b1, W2, b2 = expert_weights(inputs, "Ws", si, False)
        for t in tokens:
            z = W1 @ xt_all[t] + b1
            v[t] += ((W2.T @ dt_all[t]) * silu_grad(z)) @ W1
    dx = []
    for t in tokens:
        S = s[t, idx[t]].sum()
        ds = np.zeros(N_r)
        common = float((a[t] * g[t]).sum())
        for k in range(K):
            ds[idx[t, k]] += (a[t][k] - common) / S
        ds += lam * shape.alpha * N_r * f / T
        dl = s[t] * (ds - float((s[t] * ds).sum()))
        dx.append(v[t] + dl @ W_r)
    res["x"] = np.array(dx).reshape(len(tokens), shape.d_model)
    return res

"""Pins of the CPU oracle against what the reference pages and mathematics fix.

Every check here is independent of the oracle's own formulas: printed
numbers (tests/golden/paper_numbers.json), brute force on tiny inputs, library
routines (torch's CPU linear/SiLU, float8 and bf16 conversions), closed forms
and structural invariants.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
from synthetic import MoEShape, DTYPE_F32, DTYPE_BF16, DTYPE_FP8, make_inputs

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "paper_numbers.json")))


def tiny(**kw):
    base = dict(name="pin", T=37, d_model=24, n_routed=6, top_k=2, d_ff=40, dtype=DTYPE_F32)
    base.update(kw)
    return MoEShape(**base)


# ---------------------------------------------------------------- routing

def test_gates_sum_to_one():
    sh = tiny(T=200, n_routed=16, top_k=4)
    rt = O.route(sh, make_inputs(sh, seed=1, route_only=True))
    assert np.all(np.abs(rt["gates"].sum(axis=1) - 1.0) < 1e-12)
    assert np.all(rt["gates"] > 0)


def _brute_topk(l, K):
    """Lexicographically smallest index set among the K-subsets of maximal
    logit sum, then ordered by descending logit / ascending index."""
    n = len(l)
    best, best_sum = None, -math.inf
    for sub in itertools.combinations(range(n), K):   # lexicographic order
        s = sum(l[i] for i in sub)
        if s > best_sum:
            best, best_sum = sub, s
    return sorted(best, key=lambda i: (-l[i], i))


@pytest.mark.parametrize("n,K", [(4, 1), (5, 2), (6, 3), (8, 2), (8, 4), (8, 8)])
def test_topk_brute_force_with_ties(n, K):
    rng = np.random.default_rng(n * 10 + K)
    l = rng.integers(-2, 3, size=(300, n)).astype(np.float64)   # many exact ties
    got = O.topk_select(l, K)
    for t in range(l.shape[0]):
        assert list(got[t]) == _brute_topk(list(l[t]), K), (t, l[t])


@pytest.mark.parametrize("entry", GOLDEN["combinations"][:2], ids=lambda e: f"C({e['n']},{e['k']})")
def test_combination_counts_by_enumeration(entry):
    n, K = entry["n"], entry["k"]
    seen = set()
    for sub in itertools.combinations(range(n), K):
        l = np.zeros((1, n))
        l[0, list(sub)] = 10.0 + np.arange(K)          # large logits on the pair
        seen.add(tuple(sorted(O.topk_select(l, K)[0])))
        assert tuple(sorted(O.topk_select(l, K)[0])) == sub
    assert len(seen) == entry["value"]


def test_combination_count_64_choose_8():
    e = GOLDEN["combinations"][2]
    assert math.comb(e["n"], e["k"]) == e["value"]
    # and the oracle reaches arbitrary 8-subsets of 64 experts
    rng = np.random.default_rng(5)
    for _ in range(200):
        sub = np.sort(rng.choice(64, 8, replace=False))
        l = rng.normal(size=(1, 64))
        l[0, sub] += 100.0
        assert np.array_equal(np.sort(O.topk_select(l, 8)[0]), sub)


def test_selection_on_logits_equals_selection_on_softmax():
    sh = tiny(T=300, n_routed=12, top_k=3)
    rt = O.route(sh, make_inputs(sh, seed=2, route_only=True))
    by_s = np.argsort(-rt["s"], axis=1, kind="stable")[:, :3]
    ok = rt["gap"] > 1e-9
    assert np.array_equal(np.sort(by_s[ok], 1), np.sort(rt["idx"][ok], 1))


# ---------------------------------------------------------------- near-tie gap
#
# topk_gap decides which tokens the end-to-end comparison leaves out (a K-th
# and (K+1)-th logit closer than 1e-5 may swap between fp32 and fp64).  It is
# the margin of the top-K choice: the K-th largest key minus the (K+1)-th,
# infinite when every expert is chosen.

@pytest.mark.parametrize("row,expect", [
    # descending 3, 1, 1, 0
    ([3.0, 1.0, 1.0, 0.0], {1: 2.0, 2: 0.0, 3: 1.0, 4: math.inf}),
    # descending 2, 2, 0.5, 0.25, -1 (unsorted, with a tie at the top)
    ([0.5, 2.0, -1.0, 2.0, 0.25], {1: 0.0, 2: 1.5, 3: 0.25, 4: 1.25, 5: math.inf}),
])
def test_topk_gap_hand_computed(row, expect):
    l = np.array([row])
    for K, g in expect.items():
        assert O.topk_gap(l, K)[0] == g, (row, K)


def test_topk_gap_is_the_margin_of_the_brute_force_choice():
    # independent of any sort: the smallest chosen key minus the largest key
    # left out, with the chosen set from the brute-force search above
    rng = np.random.default_rng(9)
    for n, K in [(5, 1), (6, 2), (7, 3), (8, 7)]:
        l = rng.normal(size=(60, n)).round(2)          # some exact ties
        got = O.topk_gap(l, K)
        for t in range(l.shape[0]):
            sel = _brute_topk(list(l[t]), K)
            rest = [i for i in range(n) if i not in sel]
            assert got[t] == min(l[t][sel]) - max(l[t][rest]), (n, K, t)


def test_route_gap_uses_the_selection_keys():
    # one token, d = 1: x = 1 and W_r = (3, 1, 1, 0) give logits 3, 1, 1, 0
    x = np.array([[1.0]])
    W_r = np.array([[3.0], [1.0], [1.0], [0.0]])
    b = np.array([-2.5, 0.0, 0.25, 0.0])
    inp = {"x": x, "W_r": W_r, "logit_bias": None}
    sh = MoEShape("gap", 1, 1, 4, 1, 8, dtype=DTYPE_F32)
    assert O.route(sh, inp)["gap"][0] == 2.0
    assert O.route(sh.replace(top_k=2), inp)["gap"][0] == 0.0
    # a bias changes the keys to 0.5, 1, 1.25, 0 in both modes: added to the
    # logits (mode 0) or to the selection keys only (mode 1)
    for mode in (0, 1):
        inp_b = dict(inp, logit_bias=b)
        r1 = O.route(sh.replace(bias_mode=mode), inp_b)
        r2 = O.route(sh.replace(bias_mode=mode, top_k=2), inp_b)
        assert list(r1["idx"][0]) == [2] and list(r2["idx"][0]) == [2, 1]
        assert r1["gap"][0] == 0.25 and r2["gap"][0] == 0.5, mode


# ---------------------------------------------------------------- dispatch plan

@pytest.mark.parametrize("cf", [0.0, 0.5, 1.0, 1.25])
def test_plan_invariants(cf):
    sh = tiny(T=257, n_routed=8, top_k=3, capacity_factor=cf)
    rt = O.route(sh, make_inputs(sh, seed=3, route_only=True))
    p = rt["plan"]
    T, K = sh.T, sh.top_k
    assert p["counts"].sum() == T * K
    assert p["kept"].sum() == p["R"] <= T * K
    C = rt["C"]
    if C is not None:
        assert np.all(p["kept"] == np.minimum(p["counts"], C))
    # bijection between kept slots and rows [0, R)
    sr = p["slot_row"].reshape(-1)
    kept = sr[sr >= 0]
    assert np.array_equal(np.sort(kept), np.arange(p["R"]))
    assert np.all(p["row_slot"][kept] == np.nonzero(sr >= 0)[0])
    # rows of each expert's segment: that expert, ascending token index
    for j in range(sh.n_routed):
        rows = np.arange(p["offsets"][j], p["offsets"][j + 1])
        slots = p["row_slot"][rows]
        assert np.all(rt["idx"].reshape(-1)[slots] == j)
        assert np.all(np.diff(slots // K) > 0)
    # a dropped slot is the expert's (C+1)-th or later selection in token order
    for t in range(T):
        for k in range(K):
            j = rt["idx"][t, k]
            earlier = int(np.sum(rt["idx"][:t] == j))
            assert (p["slot_row"][t, k] < 0) == (C is not None and earlier >= C)


def test_capacity_keeps_first_C_tokens():
    sh = tiny(T=50, n_routed=4, top_k=1, capacity_factor=1.0)
    inp = make_inputs(sh, seed=4)
    inp["W_r"] = torch.zeros_like(inp["W_r"])
    inp["W_r"][0] = 1.0
    inp["x"] = torch.abs(inp["x"]) + 0.1            # every token prefers expert 0
    rt = O.route(sh, inp)
    C = rt["C"]
    assert C == math.ceil(50 * 1 / 4)
    assert np.all(rt["idx"][:, 0] == 0)
    kept = rt["plan"]["slot_row"][:, 0] >= 0
    assert np.array_equal(np.nonzero(kept)[0], np.arange(C))
    out = O.layer_forward(sh, inp, routing=rt)["out"]
    assert np.all(out[C:] == 0.0)                   # dropped, no shared expert
    assert np.all(np.abs(out[:C]).sum(axis=1) > 0)


# ---------------------------------------------------------------- expert FFN

def _torch_ffn(x, W1, b1, W2, b2):
    return F.linear(F.silu(F.linear(x, W1, b1)), W2, b2)


def test_dense_limit_single_expert():
    sh = tiny(T=33, d_model=48, n_routed=1, top_k=1, d_ff=80)
    inp = make_inputs(sh, seed=6)
    out = O.layer_forward(sh, inp)["out"]
    x = inp["x"].double()
    ref = _torch_ffn(x, inp["W1"][0].double(), inp["b1"][0].double(),
                     inp["W2"][0].double(), inp["b2"][0].double()).numpy()
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_shared_only_is_sum_of_dense_ffns():
    sh = tiny(T=20, n_routed=1, top_k=1, n_shared=3, d_ff_shared=16)
    inp = make_inputs(sh, seed=7)
    inp["W1"] = torch.zeros_like(inp["W1"])
    inp["b1"] = torch.zeros_like(inp["b1"])
    inp["W2"] = torch.zeros_like(inp["W2"])
    inp["b2"] = torch.zeros_like(inp["b2"])            # routed expert contributes 0
    out = O.layer_forward(sh, inp)["out"]
    x = inp["x"].double()
    ref = sum(_torch_ffn(x, inp["Ws1"][s].double(), inp["bs1"][s].double(),
                         inp["Ws2"][s].double(), inp["bs2"][s].double()) for s in range(3))
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_matches_dense_masked_module_form():
    """Every expert on every token, then masked by the selection and weighted
    by the renormalised top-K scores, plus the shared experts: the layer of
    the reference module, written here in torch fp64 on the CPU."""
    sh = tiny(T=41, d_model=32, n_routed=7, top_k=3, d_ff=24, n_shared=2, d_ff_shared=20)
    inp = make_inputs(sh, seed=8)
    out = O.layer_forward(sh, inp)["out"]
    x = inp["x"].double()
    scores = torch.softmax(x @ inp["W_r"].double().T, dim=-1)
    top_s, top_i = torch.topk(scores, sh.top_k, dim=-1)
    top_s = top_s / top_s.sum(-1, keepdim=True)
    ref = torch.zeros_like(x)
    for s in range(sh.n_shared):
        ref += _torch_ffn(x, inp["Ws1"][s].double(), inp["bs1"][s].double(),
                          inp["Ws2"][s].double(), inp["bs2"][s].double())
    for k in range(sh.top_k):
        for e in range(sh.n_routed):
            mask = (top_i[:, k] == e).double()[:, None]
            ref += top_s[:, k:k + 1] * mask * _torch_ffn(
                x, inp["W1"][e].double(), inp["b1"][e].double(),
                inp["W2"][e].double(), inp["b2"][e].double())
    assert np.allclose(out, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_k_equals_n_is_softmax_mixture():
    sh = tiny(T=19, n_routed=5, top_k=5)
    inp = make_inputs(sh, seed=9)
    res = O.layer_forward(sh, inp)
    x = inp["x"].double()
    s = torch.softmax(x @ inp["W_r"].double().T, dim=-1)
    ref = sum(s[:, e:e + 1] * _torch_ffn(x, inp["W1"][e].double(), inp["b1"][e].double(),
                                         inp["W2"][e].double(), inp["b2"][e].double())
              for e in range(5))
    assert np.allclose(res["out"], ref.numpy(), rtol=1e-11, atol=1e-12)


def test_active_parameter_fraction():
    g = GOLDEN["active_fraction"][0]
    N, K = g["n_experts"], g["top_k"]
    sh = tiny(T=1, d_model=16, n_routed=N, top_k=K, d_ff=24)
    inp = make_inputs(sh, seed=10)
    rt = O.route(sh, inp)
    per_expert = sum(int(inp[k][0].numel()) for k in ("W1", "b1", "W2", "b2"))
    touched = len(set(rt["idx"][0].tolist())) * per_expert
    total = sh.n_routed * per_expert
    assert touched / total == pytest.approx(g["value"], abs=0)
    # fine-grained split keeps the active parameters: K*d_ff == mK*(d_ff/m)
    fg = GOLDEN["fine_grained_split"][0]
    assert fg["K"] * fg["d_ff"] == (fg["m"] * fg["K"]) * (fg["d_ff"] // fg["m"])
    assert math.comb(fg["m"] * fg["N"], fg["m"] * fg["K"]) == GOLDEN["combinations"][2]["value"]


# ---------------------------------------------------------------- balance

def test_balance_uniform_routing_gives_alpha():
    """Cyclic logits: token t sees v rotated by t, so over N_r tokens every
    expert gets the same load and the same mean score; L must equal alpha."""
    N, K = 8, 2
    v = np.array([3.0, 2.5, 1.0, 0.5, 0.0, -0.5, -1.0, -2.0])
    l = np.stack([np.roll(v, t) for t in range(N)])
    s = O.softmax(l)
    idx = O.topk_select(l, K)
    plan = O.dispatch_plan(idx, N, None)
    alpha = GOLDEN["balance_alpha"]["value"]
    f, P, L = O.balance_stats(plan["counts"], s, K, alpha)
    assert np.allclose(f, 1.0 / N, atol=0)
    assert np.allclose(P, 1.0 / N, atol=1e-15)
    assert L == pytest.approx(alpha, rel=1e-14)


def test_balance_collapsed_router_gives_alpha_times_n():
    N, T = 16, 64
    l = np.zeros((T, N))
    l[:, 3] = 200.0                                  # one expert takes everything
    s = O.softmax(l)
    plan = O.dispatch_plan(O.topk_select(l, 1), N, None)
    f, P, L = O.balance_stats(plan["counts"], s, 1, 0.01)
    assert f[3] == 1.0 and P[3] == pytest.approx(1.0, abs=1e-15)
    assert L == pytest.approx(0.01 * N, rel=1e-14)


# ---------------------------------------------------------------- number formats

def test_e4m3_round_matches_torch():
    rng = np.random.default_rng(11)
    v = np.concatenate([
        rng.uniform(-448, 448, 20000),
        rng.uniform(-2.0 ** -5, 2.0 ** -5, 20000),          # subnormal range
        O.e4m3_decode(np.arange(256, dtype=np.uint8)),      # exact codes
    ]).astype(np.float32)
    v = v[np.isfinite(v)]
    # exact midpoints between neighbouring codes (ties to even)
    pos = O.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    v = np.concatenate([v, mids, -mids])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_round(v.astype(np.float64))
    assert np.array_equal(got, ref)
    # tiny negative values round to negative zero, tiny positive ones to zero
    assert O.e4m3_round(np.array([-1e-9, 1e-9, -0.0, 0.0])).tolist() == [0x80, 0x00, 0x80, 0x00]


def test_e4m3_saturates_and_round_trips():
    assert O.e4m3_round(np.array([1e6, -1e6, 448.0, 464.0])).tolist() == [0x7E, 0xFE, 0x7E, 0x7E]
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    assert np.array_equal(O.e4m3_round(O.e4m3_decode(codes)), codes)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(12)
    v = np.concatenate([rng.normal(size=50000), rng.normal(size=5000) * 1e-30,
                        rng.normal(size=5000) * 1e20]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.bf16_round(v.astype(np.float64)), ref)


def test_pow2_scale_is_smallest_power_of_two():
    rng = np.random.default_rng(13)
    a = np.concatenate([rng.uniform(1e-6, 1e4, 5000), 448.0 * np.exp2(np.arange(-20, 20)),
                        np.nextafter(448.0 * np.exp2(np.arange(-20, 20)), np.inf)])
    s = O.pow2_scale(a)
    k = np.log2(s)
    assert np.all(k == np.round(k))
    assert np.all(a / s <= 448.0) and np.all(a / (s / 2) > 448.0)
    assert O.pow2_scale(np.array([0.0]))[0] == 1.0


def test_pow2_scale_stays_a_normal_fp32_value():
    # amax = 448 * 2^-126 is the smallest block maximum whose own scale, 2^-126,
    # is still a normal fp32 number; below it the scale stays at 2^-126
    edge = 448.0 * 2.0 ** -126
    tiny = np.array([edge, edge / 2, 1e-37, 2.0 ** -149, np.nextafter(edge, np.inf)])
    s = O.pow2_scale(tiny)
    assert list(s[:4]) == [2.0 ** -126] * 4
    assert s[4] == 2.0 ** -125
    # the stored scale survives a round trip through fp32 unchanged
    assert np.array_equal(s.astype(np.float32).astype(np.float64), s)
    # codes of a tiny block are the values over 2^-126, rounded to e4m3
    v = np.full((1, 128), 1e-37)
    codes, sc = O.quantize_rows_1x128(v)
    assert sc[0, 0] == 2.0 ** -126
    assert np.all(O.e4m3_decode(codes) == O.e4m3_decode(O.e4m3_round(np.array([1e-37 * 2.0 ** 126])))[0])


def test_fp8_quantised_row_error_bound():
    """Per-row/128 e4m3 with a power-of-two scale: every element is within half
    a unit of the e4m3 grid at its magnitude: relative error <= 2^-4 for
    normals, absolute <= 2^-10 * scale in the subnormal range."""
    rng = np.random.default_rng(14)
    v = rng.normal(size=(64, 512))
    codes, sc = O.quantize_rows_1x128(v)
    back = O.dequant_rows_1x128(codes, sc)
    scale_full = np.repeat(sc, 128, axis=1)
    err = np.abs(back - v)
    bound = np.maximum(np.abs(v) * 2.0 ** -4, 2.0 ** -10 * scale_full)
    assert np.all(err <= bound + 1e-300)
    assert np.all(np.abs(back) <= 448.0 * scale_full)


def test_fp8_layer_dense_limit():
    """FP8 workload with one expert: the oracle equals torch's CPU linear/SiLU
    on the dequantised operands, with h re-quantised and outputs rounded to
    bf16 (checked with torch's own float8/bf16 conversions)."""
    sh = MoEShape("pin8", 16, 256, 1, 1, 128, dtype=DTYPE_FP8)
    inp = make_inputs(sh, seed=15)
    out = O.layer_forward(sh, inp)["out"]

    def q_rows(v):       # torch restatement of the 1x128 power-of-two quantiser
        vb = v.reshape(v.shape[0], -1, 128)
        amax = vb.abs().amax(-1)
        m, e = torch.frexp(amax)
        sc = torch.ldexp(torch.ones_like(amax), e - 9 + (m > 0.875).long())
        q = (vb / sc[..., None]).float().to(torch.float8_e4m3fn).double()
        return (q * sc[..., None]).reshape(v.shape)

    def deq_w(c, s):
        vals = c.view(torch.float8_e4m3fn).double()
        return vals * s.double().repeat_interleave(128, 0).repeat_interleave(128, 1)

    x = q_rows(inp["x"].double())
    h = F.silu(F.linear(x, deq_w(inp["W1"][0], inp["W1_scales"][0]), inp["b1"][0].double()))
    y = F.linear(q_rows(h), deq_w(inp["W2"][0], inp["W2_scales"][0]), inp["b2"][0].double())
    y = y.to(torch.bfloat16).double()   # single rounding: y is one expert with gate 1
    assert np.array_equal(out, y.numpy())


@pytest.mark.parametrize("T,K,N,cf,expected", [
    (8192, 8, 64, 1.25, 1280),   # DeepSeekMoE-style workload: 1.25 * 8192 * 8 / 64 exactly
    (203, 2, 6, 1.0, 68),        # 406 / 6 = 67.67 -> 68
    (777, 2, 8, 1.1, 214),       # fp32(1.1) = 1.10000002384...; * 194.25 = 213.675 -> 214
    (6, 1, 3, 0.5, 1),           # exactly 1: no rounding up
    (10, 1, 1, 0.1, 2),          # fp32(0.1) = 0.10000000149... > 0.1: 1.0000000149 -> 2
    (64, 2, 8, 0.0, None),       # no capacity limit
    (64, 2, 8, -1.0, None),
])
def test_capacity_hand_computed_values(T, K, N, cf, expected):
    """[TopK] §解決策2: C = ceil(cf * T * K / N_r) on the fp32 value of cf
    (the value the C interface receives); expected values worked by hand."""
    assert O.capacity_of(T, K, N, cf) == expected


# ---------------------------------------------------------------------------
# Selection-only bias ([TopK] §解決策3: auxiliary-loss-free balancing steers
# the choice of experts with a per-expert bias without changing the loss).


def _one_token(bias, mode):
    from synthetic import MoEShape
    sh = MoEShape("t", 1, 1, 4, 2, 64, bias_mode=mode, dtype=0)
    inp = {"x": np.array([[1.0]]), "W_r": np.array([[2.0], [1.0], [0.0], [-1.0]]),
           "logit_bias": None if bias is None else np.asarray(bias, np.float64)}
    return O.route(sh, inp)


def test_selection_bias_hand_computed():
    """l = [2, 1, 0, -1], b = [0, 0, 0, 10]: expert 3 is chosen first
    (key 9), expert 0 second (key 2); the gates come from the unbiased
    softmax: g = [e^-1, e^2] / (e^-1 + e^2) = [1/(1+e^3), e^3/(1+e^3)]."""
    r = _one_token([0.0, 0.0, 0.0, 10.0], 1)
    assert r["idx"].tolist() == [[3, 0]]
    assert r["gates"][0, 0] == pytest.approx(0.04742587317756678, rel=1e-14)
    assert r["gates"][0, 1] == pytest.approx(0.9525741268224334, rel=1e-14)
    # P is the unbiased softmax of the single token
    e = np.exp(np.array([2.0, 1.0, 0.0, -1.0]))
    assert np.allclose(r["P"], e / e.sum(), rtol=0, atol=1e-15)


def test_logit_bias_mode_uses_biased_softmax():
    """Same numbers with the bias in the logits: keys and softmax both see
    l + b = [2, 1, 0, 9], so g = [e^9, e^2] / (e^9 + e^2)."""
    r = _one_token([0.0, 0.0, 0.0, 10.0], 0)
    assert r["idx"].tolist() == [[3, 0]]
    assert r["gates"][0, 0] == pytest.approx(1.0 / (1.0 + math.exp(-7.0)), rel=1e-14)


def test_selection_bias_zero_changes_nothing():
    a = _one_token([0.0, 0.0, 0.0, 0.0], 1)
    b = _one_token(None, 0)
    assert a["idx"].tolist() == b["idx"].tolist() == [[0, 1]]
    assert np.array_equal(a["gates"], b["gates"]) and np.array_equal(a["P"], b["P"])


# ---------------------------------------------------------------------------
# Capacity variants ([TopK] §解決策2 and FAQ Q2).


def test_slot_major_priority_hand_worked():
    """idx = [[1, 0], [0, 1], [0, 1]], C = 2.  Token order keeps the first two
    tokens of each expert; slot-major keeps every first choice before any
    second choice, so expert 0 drops token 0's second choice instead of
    token 2's first."""
    idx = np.array([[1, 0], [0, 1], [0, 1]])
    tok = O.dispatch_plan(idx, 2, 2, "token")
    slot = O.dispatch_plan(idx, 2, 2, "slot")
    assert tok["slot_row"].tolist() == [[2, 0], [1, 3], [-1, -1]]
    assert slot["slot_row"].tolist() == [[2, -1], [0, 3], [1, -1]]
    assert tok["counts"].tolist() == slot["counts"].tolist() == [3, 3]
    assert slot["row_slot"].tolist() == [2, 4, 0, 3]


def test_overflow_passthrough_with_zero_experts():
    """All expert weights and biases zero: every kept slot contributes 0, so
    with pass-through the output is exactly the sum over dropped slots of
    g * x (here K = 1, g = 1, C = 1: tokens 1 and 2 come out as their input)."""
    from synthetic import MoEShape
    x = np.array([[1.0, -2.0], [0.5, 3.0], [-1.5, 0.25]])
    inp = {"x": x, "W_r": np.array([[1.0, 0.0]]), "logit_bias": None,
           "W1": np.zeros((1, 64, 2)), "b1": np.zeros((1, 64)), "W2": np.zeros((1, 2, 64)), "b2": np.zeros((1, 2)),
           "W1_scales": None, "W2_scales": None}
    cf = 0.25                                   # 0.25 * 3 = 0.75 -> C = 1
    for mode, expect in ((0, np.zeros_like(x)), (1, np.array([[0.0, 0.0], [0.5, 3.0], [-1.5, 0.25]]))):
        sh = MoEShape("p", 3, 2, 1, 1, 64, capacity_factor=cf, dtype=0, overflow_mode=mode)
        assert O.capacity_of(3, 1, 1, cf) == 1
        out = O.layer_forward(sh, inp)["out"]
        assert np.array_equal(out, expect), (mode, out)

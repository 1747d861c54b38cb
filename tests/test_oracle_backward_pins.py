"""Pins of the oracle's layer backward (CPU only).

The backward is the derivative of the forward the oracle computes; the pages
print the forward alone ("論文解説: DeepSeekMoE" §共有エキスパート機構,
§ルーティングとバランス損失, §アルゴリズム; "Sparse MoE Top-Kルーティング"
§解決策2).  It is pinned here against things other than its own formulas:

  * central differences of the forward oracle's objective
    J = <dout, out> + lam * L_balance, element by element over every input
    and weight of tiny layers, with the routing (top-K, capacity plan) checked
    to be the same at every perturbed point;
  * closed forms: with K = 1 every gate is 1, so without the balance loss the
    router gets no gradient at all; with dout = 0 only the balance loss acts
    and every expert gradient is exactly zero; with K = N_r and no capacity
    the gates are the softmax itself, so dJ/dl is the softmax Jacobian applied
    to <dout, y_j>.
"""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from oracle import moe_oracle as O  # noqa: E402
from synthetic import DTYPE_F32, MoEShape, make_inputs  # noqa: E402

EPS = 1e-5
LAM = 50.0          # makes the balance-loss term large against the tolerance


def _inputs64(shape, seed):
    inp = make_inputs(shape, seed=seed, device="cpu")
    return {k: (None if v is None else O.to_f64(v).copy()) for k, v in inp.items()}


def _objective(shape, inp, dout, lam):
    fw = O.layer_forward(shape, inp)
    rt = fw["routing"]
    return float((dout * fw["out"]).sum()) + lam * rt["loss"], rt


def _same_routing(a, b):
    return (np.array_equal(a["idx"], b["idx"])
            and np.array_equal(a["plan"]["slot_row"], b["plan"]["slot_row"]))


def _fd_check(shape, seed, lam=LAM, keys=None):
    inp = _inputs64(shape, seed)
    rng = np.random.default_rng(seed + 1000)
    dout = rng.standard_normal((shape.T, shape.d_model))
    _, rt0 = _objective(shape, inp, dout, lam)
    an = O.layer_backward(shape, inp, dout, lam=lam)
    keys = keys or ["x", "W_r", "logit_bias", "W1", "b1", "W2", "b2", "Ws1", "bs1", "Ws2", "bs2"]
    checked = 0
    for key in keys:
        if inp.get(key) is None:
            assert an.get(key) is None
            continue
        arr = inp[key]
        g = an[key]
        assert g.shape == arr.shape, key
        for i in np.ndindex(arr.shape):
            v = arr[i]
            arr[i] = v + EPS
            jp, rp = _objective(shape, inp, dout, lam)
            arr[i] = v - EPS
            jm, rm = _objective(shape, inp, dout, lam)
            arr[i] = v
            assert _same_routing(rp, rt0) and _same_routing(rm, rt0), (key, i)
            fd = (jp - jm) / (2 * EPS)
            assert abs(fd - g[i]) <= 1e-6 * max(1.0, abs(fd)), (key, i, fd, g[i])
            checked += 1
    return rt0, an, checked


def test_fd_capacity_drop_shared_expert_logit_bias():
    # C = ceil(0.75 * 6 * 2 / 4) = 3 per expert; the decode-style bias enters the logits
    sh = MoEShape("bw1", 6, 5, 4, 2, 3, n_shared=1, d_ff_shared=2, capacity_factor=0.75,
                  dtype=DTYPE_F32, zipf_logit_bias=True)
    rt, an, n = _fd_check(sh, seed=3)
    assert rt["C"] == 3
    assert (rt["plan"]["slot_row"] < 0).any(), "the case must drop a slot"
    assert n > 150
    # a dropped slot contributes nothing: its gate gradient is zero
    assert np.all(an["dgates"][rt["plan"]["slot_row"] < 0] == 0.0)


def test_fd_passthrough_slot_major():
    sh = MoEShape("bw2", 6, 5, 4, 2, 3, capacity_factor=0.75, dtype=DTYPE_F32,
                  capacity_priority=1, overflow_mode=1)
    rt, an, _ = _fd_check(sh, seed=3)
    dropped = rt["plan"]["slot_row"] < 0
    assert dropped.any()
    # a passed-through slot's gate gradient is <dout_t, x_t>, not zero
    assert np.all(an["dgates"][dropped] != 0.0)


def test_fd_selection_only_bias():
    sh = MoEShape("bw3", 7, 4, 5, 2, 3, dtype=DTYPE_F32, bias_mode=1, selection_bias=True)
    _, an, _ = _fd_check(sh, seed=5)
    assert np.all(an["logit_bias"] == 0.0)        # the bias only picks experts


def test_fd_k_equals_n():
    sh = MoEShape("bw4", 5, 4, 3, 3, 2, n_shared=1, d_ff_shared=3, dtype=DTYPE_F32)
    _fd_check(sh, seed=7)


def test_k1_router_gets_only_the_balance_gradient():
    sh = MoEShape("bw5", 6, 5, 4, 1, 3, dtype=DTYPE_F32)
    inp = _inputs64(sh, 11)
    dout = np.random.default_rng(0).standard_normal((sh.T, sh.d_model))
    an = O.layer_backward(sh, inp, dout, lam=0.0)
    assert np.all(an["W_r"] == 0.0) and np.all(an["dlogits"] == 0.0)
    # and the central differences agree, balance loss included
    _fd_check(sh, seed=11)


def test_balance_loss_alone_leaves_experts_untouched():
    sh = MoEShape("bw6", 6, 5, 4, 2, 3, n_shared=1, d_ff_shared=2, dtype=DTYPE_F32)
    inp = _inputs64(sh, 13)
    an = O.layer_backward(sh, inp, np.zeros((sh.T, sh.d_model)), lam=1.0)
    for k in ("W1", "b1", "W2", "b2", "Ws1", "bs1", "Ws2", "bs2"):
        assert np.all(an[k] == 0.0), k
    assert np.abs(an["W_r"]).max() > 0.0
    # dJ/ds_tj = alpha N_r f_j / T for every token, the closed form of dP_j/ds_tj = 1/T
    rt = O.route(sh, inp)
    assert np.allclose(an["ds"], sh.alpha * sh.n_routed * rt["f"][None, :] / sh.T, rtol=0, atol=1e-15)


def test_k_equals_n_gates_are_the_softmax():
    # with every expert selected and nothing dropped, g = s, so dJ/dl is the
    # softmax Jacobian s_i (a_i - sum_j s_j a_j) applied to a_j = <dout, y_j>
    sh = MoEShape("bw7", 5, 4, 3, 3, 2, dtype=DTYPE_F32)
    inp = _inputs64(sh, 17)
    dout = np.random.default_rng(1).standard_normal((sh.T, sh.d_model))
    an = O.layer_backward(sh, inp, dout, lam=0.0)
    rt = O.route(sh, inp)
    s, idx = rt["s"], rt["idx"]
    x = inp["x"]
    a = np.zeros_like(s)
    for j in range(sh.n_routed):
        W1, b1, W2, b2 = O.expert_weights(inp, "W", j, False)
        a[:, j] = np.einsum("td,td->t", dout, O.expert_ffn(x, W1, b1, W2, b2))
    dl = s * (a - (s * a).sum(axis=1, keepdims=True))
    assert np.allclose(an["dlogits"], dl, rtol=1e-12, atol=1e-14)
    assert np.array_equal(np.sort(idx, axis=1), np.tile(np.arange(3), (sh.T, 1)))


def test_fp8_backward_is_not_defined():
    sh = MoEShape("bw8", 4, 128, 2, 1, 128, dtype=2)
    with pytest.raises(ValueError):
        O.layer_backward(sh, {}, np.zeros((4, 128)))


def test_planted_mistakes_fail_the_central_differences(monkeypatch):
    # the pins catch a dropped balance term and a wrong SiLU derivative
    sh = MoEShape("bw9", 6, 5, 4, 2, 3, dtype=DTYPE_F32)
    real = O.silu_grad
    monkeypatch.setattr(O, "silu_grad", lambda z: 1.0 / (1.0 + np.exp(-z)))
    with pytest.raises(AssertionError):
        _fd_check(sh, seed=19, keys=["W1"])
    monkeypatch.setattr(O, "silu_grad", real)
    orig = O.layer_backward

    def no_balance(shape, inputs, dout, lam=1.0, routing=None):
        return orig(shape, inputs, dout, lam=0.0, routing=routing)

    monkeypatch.setattr(O, "layer_backward", no_balance)
    with pytest.raises(AssertionError):
        _fd_check(sh, seed=19, keys=["W_r"])


@pytest.mark.parametrize("case", ["shared-capacity-pass", "bias-f32"])
def test_sampled_backward_equals_the_full_one(case):
    """layer_backward_sample (the full-size checks' oracle) gives exactly the
    selected entries of layer_backward, which the finite differences above
    pin: selected weight-gradient rows and blocks, bias entries and dx rows."""
    if case == "shared-capacity-pass":
        sh = MoEShape("sb1", 40, 64, 6, 2, 128, n_shared=2, d_ff_shared=64, capacity_factor=0.6,
                      overflow_mode=1, dtype=1)
    else:
        sh = MoEShape("sb2", 30, 64, 5, 2, 128, zipf_logit_bias=True, dtype=DTYPE_F32)
    inp = _inputs64(sh, 3)
    rng = np.random.default_rng(11)
    dout = rng.standard_normal((sh.T, sh.d_model))
    rt = O.route(sh, inp)
    full = O.layer_backward(sh, inp, dout, lam=LAM, routing=rt)
    experts, f_idx, c_idx, tokens = [0, 2, sh.n_routed - 1], [0, 5, 127], [1, 63], [0, 7, sh.T - 1]
    fs_idx = [0, 63]
    smp = O.layer_backward_sample(sh, inp, dout, LAM, rt, experts, f_idx, c_idx, tokens, fs_idx=fs_idx)

    def close(a, b):
        assert np.allclose(a, b, rtol=1e-11, atol=1e-11 * (1.0 + np.abs(b).max()))

    for e in experts:
        close(smp["W1"][e], full["W1"][e][f_idx])
        close(smp["b1"][e], full["b1"][e][f_idx])
        close(smp["W2"][e], full["W2"][e][np.ix_(c_idx, f_idx)])
        close(smp["b2"][e], full["b2"][e][c_idx])
    for si in range(sh.n_shared):
        close(smp["Ws1"][si], full["Ws1"][si][fs_idx])
        close(smp["bs1"][si], full["bs1"][si][fs_idx])
        close(smp["Ws2"][si], full["Ws2"][si][np.ix_(c_idx, fs_idx)])
        close(smp["bs2"][si], full["bs2"][si][c_idx])
    close(smp["x"], full["x"][tokens])
    # the case reaches a dropped slot passed through and an expert with several rows
    if case == "shared-capacity-pass":
        assert (rt["plan"]["slot_row"] == -1).any()

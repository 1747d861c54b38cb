"""GPU parity of the layer backward (moe_layer_backward) against the oracle's
layer_backward, on the product's own forward results.

The forward runs through its stage entry points; the oracle's routing is
taken on the product's fp32 logits (checked bit-exact), so both sides use the
same top-K choice and capacity plan.  Every gradient is compared by relative
Frobenius error: 1e-4 for fp32 layers, 1e-2 for bf16 (the gate gradients
read the product's bf16 expert outputs, whose rounding of h and y puts them
about 2e-3 from the oracle's fp64 values; the bf16 expert GEMMs run on the
tensor cores on bf16 copies of dy, SiLU(z), SiLU'(z) and dz, each rounding
about 1e-3), and each row of every gradient (a weight gradient's row is one
output unit's weights) within 4x that bound, relative to the larger of its
own norm and the gradient's median row norm (a row of an expert with three
tokens whose terms nearly cancel sits far below the typical row, and the
bf16 roundings of its operands set its error on the typical row's scale).  The bf16 cases span several
128-row and 256-column tiles with ragged tails, experts no token reaches
(their gradients must be exact zeros) and shared experts of a width that is
not a multiple of the tile."""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_20_b200 as M
from synthetic import DTYPE_BF16, DTYPE_F32, MoEShape

from moe_testlib import ROW_FACTOR, cpu, gpu_inputs, rel_frob, row_err_scaled_max, run_stages

pytestmark = pytest.mark.gpu

TOL = {DTYPE_F32: 1e-4, DTYPE_BF16: 1e-2}

CASES = {
    "f32-cap-shared-bias": MoEShape("k1", 100, 128, 6, 2, 64, n_shared=1, d_ff_shared=64, capacity_factor=0.7,
                                    dtype=DTYPE_F32, zipf_logit_bias=True),
    "bf16-pass-slot": MoEShape("k2", 150, 128, 8, 2, 128, capacity_factor=0.8, dtype=DTYPE_BF16,
                               capacity_priority=1, overflow_mode=1),
    "bf16-selbias-shared": MoEShape("k3", 96, 128, 16, 4, 128, n_shared=2, d_ff_shared=64, dtype=DTYPE_BF16,
                                    bias_mode=1, selection_bias=True),
    "f32-k-equals-n": MoEShape("k4", 40, 128, 4, 4, 128, dtype=DTYPE_F32),
    "bf16-e64-k8": MoEShape("k5", 64, 128, 64, 8, 128, dtype=DTYPE_BF16),
    # several m-tiles per expert, n-tails of 128 (d = 384, d_ff = 640), two
    # shared experts of width 192, a capacity that drops slots
    "bf16-tiles-shared-cap": MoEShape("k6", 600, 384, 8, 2, 640, n_shared=2, d_ff_shared=192,
                                      capacity_factor=1.1, dtype=DTYPE_BF16),
    # most of the 64 experts get no token: zero weight gradients
    "bf16-empty-experts": MoEShape("k7", 40, 128, 64, 1, 192, dtype=DTYPE_BF16),
    # an expert segment longer than one 64-row k-block many times over,
    # d_ff two tiles and a half, pass-through on
    "bf16-long-segments": MoEShape("k8", 1100, 256, 4, 2, 576, capacity_factor=0.9, dtype=DTYPE_BF16,
                                   overflow_mode=1),
    # d_model = 320 (K and N tails of 64 in every GEMM that spans d), a
    # shared expert
    "bf16-d320-shared": MoEShape("k9", 200, 320, 8, 2, 192, n_shared=1, d_ff_shared=128, dtype=DTYPE_BF16),
}


def _grad_buffers(shape, inp, dev):
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"dx": torch.empty((shape.T, shape.d_model), **f32),
         "dW_r": torch.empty(inp["W_r"].shape, **f32),
         "dW1": torch.empty(inp["W1"].shape, **f32), "db1": torch.empty(inp["b1"].shape, **f32),
         "dW2": torch.empty(inp["W2"].shape, **f32), "db2": torch.empty(inp["b2"].shape, **f32)}
    if inp["logit_bias"] is not None:
        g["d_logit_bias"] = torch.empty(shape.n_routed, **f32)
    if shape.n_shared:
        for k in ("Ws1", "bs1", "Ws2", "bs2"):
            g["d" + k] = torch.empty(inp[k].shape, **f32)
    for v in g.values():
        v.fill_(float("nan"))                 # every gradient must be written in full
    return g


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(name):
    sh = CASES[name]
    lam = 5.0
    inp = gpu_inputs(sh, seed=1)
    o = run_stages(sh, inp, logits=True)
    assert o["status"] == 0
    dev = inp["x"].device
    gen = torch.Generator().manual_seed(7)
    dout = torch.randn((sh.T, sh.d_model), generator=gen).to(inp["x"].dtype).to(dev)
    grads = _grad_buffers(sh, inp, dev)
    tensors = {k: inp[k] for k in ("x", "W_r", "W1", "b1", "W2", "b2", "Ws1", "bs1", "Ws2", "bs2")}
    tensors.update({k: o[k] for k in ("logits", "topk_idx", "gates", "counts", "offsets", "slot_row",
                                      "row_slot", "x_disp", "y")})
    tensors["dout"] = dout
    tensors.update(grads)
    cfg = o["cfg"]
    bws = torch.empty(M.moe_backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    before = M.moe_kernel_launches()
    M.moe_layer_backward(cfg, lam, tensors, bws)
    torch.cuda.synchronize()
    assert M.moe_kernel_launches() > before
    assert bws[:4].view(torch.int32).item() == 0             # device status word: no timeout

    inp_cpu = {k: cpu(v) for k, v in inp.items()}
    rt = O.route(sh, inp_cpu, logits=cpu(o["logits"]).double().numpy())
    assert np.array_equal(rt["idx"], cpu(o["topk_idx"]).numpy())
    assert np.array_equal(rt["plan"]["slot_row"], cpu(o["slot_row"]).numpy())
    ref = O.layer_backward(sh, inp_cpu, O.to_f64(cpu(dout)), lam=lam, routing=rt)
    for k, v in grads.items():
        got = cpu(v).double().numpy()
        assert np.isfinite(got).all(), k
        want = ref["logit_bias" if k == "d_logit_bias" else k[1:]]
        if np.linalg.norm(want) == 0.0:
            assert np.all(got == 0.0), k                 # e.g. a selection-only bias
            continue
        assert rel_frob(got, want) < TOL[sh.dtype], (k, rel_frob(got, want))
        if got.ndim >= 2:
            g2 = got.reshape(-1, got.shape[-1])
            w2 = want.reshape(-1, want.shape[-1])
            zero = np.linalg.norm(w2, axis=1) == 0.0
            assert np.all(g2[zero] == 0.0), (k, "rows of untouched experts")
            r = row_err_scaled_max(g2[~zero], w2[~zero])
            assert r < ROW_FACTOR * TOL[sh.dtype], (k, "worst row", r)


def test_backward_is_deterministic():
    sh = CASES["bf16-pass-slot"]
    inp = gpu_inputs(sh, seed=2)
    o = run_stages(sh, inp, logits=True)
    dev = inp["x"].device
    dout = torch.randn((sh.T, sh.d_model), generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).to(dev)
    runs = []
    for _ in range(2):
        grads = _grad_buffers(sh, inp, dev)
        tensors = {k: inp[k] for k in ("x", "W_r", "W1", "b1", "W2", "b2")}
        tensors.update({k: o[k] for k in ("logits", "topk_idx", "gates", "counts", "offsets", "slot_row",
                                          "row_slot", "x_disp", "y")})
        tensors["dout"] = dout
        tensors.update(grads)
        bws = torch.empty(M.moe_backward_workspace_size(o["cfg"]), dtype=torch.uint8, device=dev)
        bws.fill_(0xA5)                                  # scratch contents must not matter
        M.moe_layer_backward(o["cfg"], 1.0, tensors, bws)
        torch.cuda.synchronize()
        runs.append({k: cpu(v) for k, v in grads.items()})
    for k in runs[0]:
        assert torch.equal(runs[0][k], runs[1][k]), k

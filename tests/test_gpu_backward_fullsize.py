"""GPU parity of moe_layer_backward at the full sizes of the two bf16
workloads (Mixtral-shaped and DeepSeekMoE-style), in the launch
configuration the benchmark times.  The oracle computes a sample of the
gradients one entry set at a time (layer_backward_sample, pinned against
the full layer_backward on small layers): for the first, the last, the most
and the least loaded routed expert, the rows of dW1 and the blocks of dW2 at
the tile edges of d_ff (0, 127, 128, 255, 256, the last 128, the last) and of
d_model plus seeded random ones, db1 and db2 at those indices; the same for
every shared expert; dx of the first, the last and seeded random tokens.
Routing comes from the product's fp32 logits on both sides (checked equal),
so both take the top-K and capacity decisions in the same precision.  The
bound is the bf16 one of the small-layer backward tests: relative Frobenius
error 1e-2 per sampled block and 4x that per row, relative to the larger of
the row's norm and the block's median row norm."""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_20_b200 as M
from synthetic import WORKLOADS

import moe_testlib as TL

TOL = 1e-2
LAM = 1.0


def _edges(n, rng, extra=6):
    base = [0, 127, 128, 255, 256, n - 128, n - 1]
    pick = rng.choice(n, size=min(n, extra), replace=False)
    return np.unique(np.clip(np.concatenate([base, pick]), 0, n - 1)).astype(np.int64)


def _check(got, want, what):
    got = np.asarray(got, np.float64).reshape(-1, np.shape(want)[-1] if np.ndim(want) > 1 else 1)
    want = np.asarray(want, np.float64).reshape(got.shape)
    if np.linalg.norm(want) == 0.0:
        assert np.all(got == 0.0), what
        return
    e = TL.rel_frob(got, want)
    assert e < TOL, (what, "rel_frob", e)
    if want.shape[1] > 1:
        r = TL.row_err_scaled_max(got, want)
        assert r < TL.ROW_FACTOR * TOL, (what, "worst row", r)


@pytest.mark.gpu
@pytest.mark.parametrize("cid", [2, 3])
def test_backward_fullsize(cid):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sh = WORKLOADS[cid]
    inp = TL.gpu_inputs(sh, seed=0, on_device_gen=True)
    o = TL.run_stages(sh, inp, logits=True)
    assert o["status"] == 0
    dev = inp["x"].device
    gen = torch.Generator(device=dev).manual_seed(100 + cid)
    dout = torch.randn((sh.T, sh.d_model), generator=gen, device=dev).to(torch.bfloat16)
    f32 = dict(dtype=torch.float32, device=dev)
    t = {k: inp.get(k) for k in ("x", "W_r", "W1", "b1", "W2", "b2", "Ws1", "bs1", "Ws2", "bs2")}
    t.update({k: o[k] for k in ("logits", "topk_idx", "gates", "counts", "offsets", "slot_row", "row_slot",
                                "x_disp", "y")})
    g = {"dx": torch.empty((sh.T, sh.d_model), **f32), "dW_r": torch.empty(inp["W_r"].shape, **f32),
         "dW1": torch.empty(inp["W1"].shape, **f32), "db1": torch.empty(inp["b1"].shape, **f32),
         "dW2": torch.empty(inp["W2"].shape, **f32), "db2": torch.empty(inp["b2"].shape, **f32)}
    if inp.get("logit_bias") is not None:
        g["d_logit_bias"] = torch.empty(sh.n_routed, **f32)
    if sh.n_shared:
        for k in ("Ws1", "bs1", "Ws2", "bs2"):
            g["d" + k] = torch.empty(inp[k].shape, **f32)
    for v in g.values():
        v.fill_(float("nan"))
    t["dout"] = dout
    t.update(g)
    bws = torch.empty(M.moe_backward_workspace_size(o["cfg"]), dtype=torch.uint8, device=dev)
    M.moe_layer_backward(o["cfg"], LAM, t, bws)
    torch.cuda.synchronize()
    assert bws[:4].view(torch.int32).item() == 0

    inp_cpu = {k: TL.cpu(v) for k, v in inp.items()}
    rt = O.route(sh, inp_cpu, logits=TL.cpu(o["logits"]).double().numpy())
    assert np.array_equal(rt["idx"], TL.cpu(o["topk_idx"]).numpy())
    assert np.array_equal(rt["plan"]["slot_row"], TL.cpu(o["slot_row"]).numpy())
    rng = np.random.default_rng(cid)
    kept = rt["plan"]["kept"]
    nz = np.flatnonzero(kept)
    experts = sorted({0, sh.n_routed - 1, int(np.argmax(kept)), int(nz[np.argmin(kept[nz])])})
    f_idx = _edges(sh.d_ff, rng)
    c_idx = _edges(sh.d_model, rng)
    fs_idx = _edges(sh.d_ff_shared, rng) if sh.n_shared else None
    tokens = np.unique(np.concatenate([[0, sh.T - 1], rng.choice(sh.T, size=6, replace=False)])).tolist()
    dout_np = O.to_f64(TL.cpu(dout))
    smp = O.layer_backward_sample(sh, inp_cpu, dout_np, LAM, rt, experts, f_idx, c_idx, tokens, fs_idx=fs_idx)

    fi, ci = torch.as_tensor(f_idx, device=dev), torch.as_tensor(c_idx, device=dev)
    for e in experts:
        _check(TL.cpu(g["dW1"][e][fi]).numpy(), smp["W1"][e], f"dW1[{e}]")
        _check(TL.cpu(g["db1"][e][fi]).numpy(), smp["b1"][e], f"db1[{e}]")
        _check(TL.cpu(g["dW2"][e][ci][:, fi]).numpy(), smp["W2"][e], f"dW2[{e}]")
        _check(TL.cpu(g["db2"][e][ci]).numpy(), smp["b2"][e], f"db2[{e}]")
    if sh.n_shared:
        fsi = torch.as_tensor(fs_idx, device=dev)
        for si in range(sh.n_shared):
            _check(TL.cpu(g["dWs1"][si][fsi]).numpy(), smp["Ws1"][si], f"dWs1[{si}]")
            _check(TL.cpu(g["dbs1"][si][fsi]).numpy(), smp["bs1"][si], f"dbs1[{si}]")
            _check(TL.cpu(g["dWs2"][si][ci][:, fsi]).numpy(), smp["Ws2"][si], f"dWs2[{si}]")
            _check(TL.cpu(g["dbs2"][si][ci]).numpy(), smp["bs2"][si], f"dbs2[{si}]")
    _check(TL.cpu(g["dx"][torch.as_tensor(tokens, device=dev)]).numpy(), smp["x"], "dx")
    # every gradient was written in full and is finite
    for k, v in g.items():
        assert bool(torch.isfinite(v).all()), k

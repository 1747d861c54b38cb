"""Helpers shared by the GPU parity tests: run every stage of the library
through the C ABI on seeded inputs, and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import sparse_mixture_experts_20_b200 as M
from synthetic import make_inputs

TOL_REL_FROB = {0: 1e-5, 1: 1e-2, 2: 3e-2}     # fp32 / bf16 / fp8 layer output
NEAR_TIE = 1e-5
# Per-row bound beside the whole-tensor one: every row's relative error must
# stay within ROW_FACTOR times the tolerance.  A whole-tensor norm over tens of
# thousands of rows hardly moves when a few rows (a ragged tail tile) are
# wrong; a row-wise bound catches them.
ROW_FACTOR = 4.0


def rel_frob(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def row_rel_max(a: np.ndarray, b: np.ndarray) -> float:
    """Largest relative error of one row: max_i |a_i - b_i| / |b_i| over rows."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if a.shape[0] == 0:
        return 0.0
    num = np.linalg.norm(a - b, axis=1)
    den = np.linalg.norm(b, axis=1)
    return float(np.max(num / np.where(den > 0, den, 1.0)))


def assert_close_rows(got, ref, tol, what=""):
    """Whole-tensor relative Frobenius error below tol and every row's
    relative error below ROW_FACTOR * tol."""
    e = rel_frob(got, ref)
    assert e < tol, (what, "rel_frob", e)
    r = row_rel_max(got, ref)
    assert r < ROW_FACTOR * tol, (what, "worst row", r)
    return e, r


def row_err_scaled_max(a: np.ndarray, b: np.ndarray) -> float:
    """Largest row error relative to max(the row's own norm, the median
    non-zero row norm of b).  A row far below the typical row of a gradient
    is a sum of few, partly cancelling terms; the bf16 roundings of the
    operands then set its error on the matrix's scale, not on its own."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if a.shape[0] == 0:
        return 0.0
    n = np.linalg.norm(b, axis=1)
    nz = n[n > 0]
    med = float(np.median(nz)) if nz.size else 1.0
    return float(np.max(np.linalg.norm(a - b, axis=1) / np.maximum(n, med)))


def gpu_inputs(shape, seed, device="cuda", on_device_gen=False):
    """Seeded inputs on the GPU.  Small shapes are drawn on the CPU and copied;
    on_device_gen draws them directly on the GPU (full-size workloads)."""
    if on_device_gen:
        return make_inputs(shape, seed, device=device)
    cpu = make_inputs(shape, seed, device="cpu")
    return {k: (None if v is None else v.to(device)) for k, v in cpu.items()}


def act_dtype(shape):
    return torch.float32 if shape.dtype == 0 else torch.bfloat16


def run_stages(shape, inp, logits=True):
    """Route -> dispatch -> expert FFN -> combine -> balance, each through its
    own entry point.  Returns every output as a CUDA tensor."""
    dev = inp["x"].device
    cfg = M.make_config(shape)
    T, K, E, d = shape.T, shape.top_k, shape.n_routed, shape.d_model
    cap, r_cap, x_rows, y_rows = M.moe_buffer_rows(cfg)
    ws = torch.empty(M.moe_workspace_size(cfg), dtype=torch.uint8, device=dev)
    M.moe_workspace_init(cfg, ws)
    o = {"cfg": cfg, "ws": ws, "capacity": cap, "r_cap": r_cap}
    i32 = dict(dtype=torch.int32, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    o["topk_idx"] = torch.empty((T, K), **i32)
    o["gates"] = torch.empty((T, K), **f32)
    o["logits"] = torch.empty((T, E), **f32) if logits else None
    M.moe_route(cfg, inp["x"], inp["W_r"], inp["logit_bias"], o["topk_idx"], o["gates"], o["logits"], ws)
    fp8 = shape.dtype == 2
    o["counts"] = torch.empty(E, **i32)
    o["kept"] = torch.empty(E, **i32)
    o["offsets"] = torch.empty(E + 1, **i32)
    o["slot_row"] = torch.empty((T, K), **i32)
    o["row_slot"] = torch.empty(max(r_cap, 1), **i32)
    o["x_disp"] = torch.empty((x_rows, d), dtype=torch.uint8 if fp8 else act_dtype(shape), device=dev)
    o["x_disp_scales"] = torch.empty((x_rows, d // 128), **f32) if fp8 else None
    M.moe_dispatch(cfg, inp["x"], o["topk_idx"], o["counts"], o["kept"], o["offsets"], o["slot_row"],
                   o["row_slot"], o["x_disp"], o["x_disp_scales"], ws)
    o["y"] = torch.empty((y_rows, d), dtype=act_dtype(shape), device=dev)
    M.moe_expert_ffn(cfg, inp["x"], o["x_disp"], o["x_disp_scales"], o["offsets"],
                     inp["W1"], inp["W1_scales"], inp["b1"], inp["W2"], inp["W2_scales"], inp["b2"],
                     inp["Ws1"], inp["Ws1_scales"], inp["bs1"], inp["Ws2"], inp["Ws2_scales"], inp["bs2"],
                     o["y"], ws)
    o["out"] = torch.empty((T, d), dtype=act_dtype(shape), device=dev)
    M.moe_combine(cfg, o["y"], o["gates"], o["slot_row"], o["out"], x=inp["x"])
    o["f"] = torch.empty(E, **f32)
    o["P"] = torch.empty(E, **f32)
    o["loss"] = torch.empty(1, **f32)
    M.moe_balance_stats(cfg, o["counts"], ws, o["f"], o["P"], o["loss"])
    torch.cuda.synchronize()
    o["status"] = M.moe_get_device_status(cfg, ws)
    return o


def run_layer(shape, inp):
    """The whole layer through moe_layer_forward."""
    cfg = M.make_config(shape)
    layer = M.MoELayer(cfg, inp, device=inp["x"].device)
    out, f, P, loss = layer.forward(inp["x"])
    torch.cuda.synchronize()
    return {"out": out, "f": f, "P": P, "loss": loss, "topk_idx": layer.topk_idx,
            "gates": layer.gates, "counts": layer.counts, "status": layer.device_status()}


def cpu(t):
    return None if t is None else t.detach().cpu()


def check_routing(shape, inp, o):
    """Routing bit-exact on the product's own fp32 logits; gates, logits, P
    and the loss within their tolerances."""
    logits = cpu(o["logits"]).double().numpy()
    rt_prod = O.route(shape, inp, logits=logits)          # selection on product logits
    idx = cpu(o["topk_idx"]).numpy()
    assert np.array_equal(idx, rt_prod["idx"]), "top-K indices differ on identical logits"
    # the product's logits against the oracle's fp64 logits
    l64 = rt_prod["logits"]
    scale = np.abs(l64).max() + 1e-30
    assert np.max(np.abs(logits - l64)) / scale < 2e-5
    # softmax, gates and P of the product's logits (the fused part of the
    # router), then P against the oracle's own fp64 logits (spec 1e-6)
    s_prod = O.softmax(logits)
    g = cpu(o["gates"]).double().numpy()
    assert np.max(np.abs(g - O.gates_of(s_prod, idx))) < 2e-6
    P = cpu(o["P"]).double().numpy()
    assert np.max(np.abs(P - s_prod.mean(axis=0))) < 1e-6
    assert np.max(np.abs(P - rt_prod["P"])) < 1e-6
    f = cpu(o["f"]).double().numpy()
    assert np.max(np.abs(f - rt_prod["f"])) < 1e-6
    assert abs(float(cpu(o["loss"])[0]) - rt_prod["loss"]) < 1e-6 * max(1.0, abs(rt_prod["loss"]))
    return rt_prod


def check_dispatch(shape, inp, o, rt_prod):
    plan = rt_prod["plan"]
    assert np.array_equal(cpu(o["counts"]).numpy(), plan["counts"])
    assert np.array_equal(cpu(o["kept"]).numpy(), plan["kept"])
    assert np.array_equal(cpu(o["offsets"]).numpy(), plan["offsets"])
    assert np.array_equal(cpu(o["slot_row"]).numpy(), plan["slot_row"])
    R = plan["R"]
    assert np.array_equal(cpu(o["row_slot"]).numpy()[:R], plan["row_slot"])
    K = shape.top_k
    src_tok = plan["row_slot"] // K
    x = cpu(inp["x"])
    if shape.dtype == 2:
        codes, sc = O.quantize_rows_1x128(O.to_f64(x))
        xd = cpu(o["x_disp"]).numpy()
        xs = cpu(o["x_disp_scales"]).double().numpy()
        assert np.array_equal(xd[:R], codes[src_tok])
        assert np.array_equal(xs[:R], sc[src_tok])
        if shape.n_shared > 0:
            rc = o["r_cap"]
            assert np.array_equal(xd[rc:rc + shape.T], codes)
            assert np.array_equal(xs[rc:rc + shape.T], sc)
    else:
        assert torch.equal(cpu(o["x_disp"])[:R], x[torch.as_tensor(src_tok, dtype=torch.long)])


def check_expert_ffn(shape, inp, o, rt_prod, rows=None, tokens=None):
    """Expert outputs of the routed rows (all, or a sample) and of the shared
    experts against the oracle's FFN on the product's own dispatched rows."""
    fp8 = shape.dtype == 2
    plan = rt_prod["plan"]
    R = plan["R"]
    y = cpu(o["y"]).double().numpy()
    tol = TOL_REL_FROB[shape.dtype]
    if fp8:
        xin = O.dequant_rows_1x128(cpu(o["x_disp"]).numpy(), cpu(o["x_disp_scales"]).double().numpy())
    else:
        xin = O.to_f64(cpu(o["x_disp"]))
    rows = np.arange(R) if rows is None else np.asarray(rows)
    offs = plan["offsets"]
    errs = []
    for e in range(shape.n_routed):
        sel = rows[(rows >= offs[e]) & (rows < offs[e + 1])]
        if len(sel) == 0:
            continue
        W1, b1, W2, b2 = O.expert_weights(inp, "W", e, fp8)
        ref = O.expert_ffn(xin[sel], W1, b1, W2, b2, fp8_hidden=fp8)
        if fp8:
            ref = O.bf16_round(ref)
        errs.append((y[sel], ref))
    if errs:
        got = np.concatenate([a for a, _ in errs])
        ref = np.concatenate([b for _, b in errs])
        assert_close_rows(got, ref, tol, "routed expert rows")
    rc = o["r_cap"]
    for s in range(shape.n_shared):
        W1, b1, W2, b2 = O.expert_weights(inp, "Ws", s, fp8)
        if fp8:
            xs = O.dequant_rows_1x128(cpu(o["x_disp"]).numpy()[rc:rc + shape.T],
                                      cpu(o["x_disp_scales"]).double().numpy()[rc:rc + shape.T])
        else:
            xs = O.to_f64(cpu(inp["x"]))
        tok = np.arange(shape.T) if tokens is None else np.asarray(tokens)
        ref = O.expert_ffn(xs[tok], W1, b1, W2, b2, fp8_hidden=fp8)
        if fp8:
            ref = O.bf16_round(ref)
        got = y[rc + s * shape.T + tok]
        assert_close_rows(got, ref, tol, f"shared expert {s}")


def check_combine(shape, o, rt_prod, x=None):
    """out[t] = sum_k g y[slot_row] (+ g x[t] for slots over the capacity with
    pass-through) + sum_s y_shared, from the product's own y, gates and
    slot_row (only rounding of the output may differ)."""
    y = cpu(o["y"]).double().numpy()
    g = cpu(o["gates"]).double().numpy()
    sr = cpu(o["slot_row"]).numpy()
    T, K = shape.T, shape.top_k
    ref = np.zeros((T, shape.d_model))
    for k in range(K):
        ok = sr[:, k] >= 0
        ref[ok] += g[ok, k:k + 1] * y[sr[ok, k]]
        if getattr(shape, "overflow_mode", 0) == 1:
            dropped = sr[:, k] == -1
            ref[dropped] += g[dropped, k:k + 1] * O.to_f64(cpu(x))[dropped]
    rc = o["r_cap"]
    for s in range(shape.n_shared):
        ref += y[rc + s * T: rc + (s + 1) * T]
    out = cpu(o["out"]).double().numpy()
    # the output's own rounding: fp32, or bf16 (half an ulp, 2^-9 per element)
    bound = 1e-6 if shape.dtype == 0 else 2.0 ** -8
    assert rel_frob(out, ref) < bound, rel_frob(out, ref)
    assert row_rel_max(out, ref) < bound, row_rel_max(out, ref)


def check_end_to_end(shape, inp, out, idx_prod, tokens=None, routing=None):
    """Layer output against the oracle's full fp64 forward, excluding near-tie
    tokens and (with a capacity) tokens whose kept set differs.  Returns the
    error and the number of excluded tokens."""
    rt = routing if routing is not None else O.route(shape, inp)
    T = shape.T
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    ok = rt["gap"][tokens] >= NEAR_TIE
    if shape.capacity_factor > 0:
        prod_plan = O.dispatch_plan(np.asarray(idx_prod), shape.n_routed, rt["C"],
                                    "slot" if getattr(shape, "capacity_priority", 0) == 1 else "token")
        same = np.all((prod_plan["slot_row"][tokens] >= 0) == (rt["plan"]["slot_row"][tokens] >= 0), axis=1)
        same &= np.all(np.sort(np.asarray(idx_prod)[tokens], 1) == np.sort(rt["idx"][tokens], 1), axis=1)
        ok &= same
    use = tokens[ok]
    ref = O.layer_forward(shape, inp, tokens=use, routing=rt)["out"]
    got = cpu(out).double().numpy()[use]
    err = rel_frob(got, ref)
    worst = row_rel_max(got, ref)
    assert worst < ROW_FACTOR * TOL_REL_FROB[shape.dtype], ("worst token", worst)
    return err, int((~ok).sum())

"""Expert parallelism on the GPU ("エキスパート並列（Expert Parallelism）"
§推論フロー; "DeepSeek DeepEP" §DeepEP とは: FP8 dispatch, bf16 combine).

moe_expert_ffn_segments runs the grouped expert FFN over caller-made
segments, the layout an expert-parallel rank receives (one segment per
source rank and expert, in arrival order): on a scrambled layout of the
dispatched rows (each expert's rows cut in two, the pieces in reverse expert
order) it must give every row exactly what moe_expert_ffn gives it (the same
tiles of K in the same order), for fp32, bf16 and FP8 layers; a segment that
names no held expert is skipped and reported.  ExpertParallelMoE on a
one-rank NCCL group runs the whole exchange path (counts and rows through
all_to_all, the segments, the outputs back, the shared experts, the
combine) and must reproduce moe_layer_forward bit for bit.  More ranks than
GPUs cannot run here; the multi-rank plan is checked on CPU (test_ep_host)."""
import datetime
import socket

import numpy as np
import pytest
import torch

import sparse_mixture_experts_20_b200 as M
from sparse_mixture_experts_20_b200 import ep
from synthetic import DTYPE_BF16, DTYPE_F32, DTYPE_FP8, MoEShape

import moe_testlib as TL

pytestmark = pytest.mark.gpu

SEG_CASES = {
    "f32": MoEShape("g1", 200, 128, 8, 2, 128, dtype=DTYPE_F32),
    "bf16": MoEShape("g2", 700, 384, 8, 2, 640, dtype=DTYPE_BF16),
    "fp8": MoEShape("g3", 300, 256, 16, 4, 256, dtype=DTYPE_FP8),
}


def _scrambled(offsets):
    """Segments of the dispatched rows: each expert's rows cut in two, the
    second halves first, experts in reverse order; returns (perm, seg_off,
    seg_exp) with perm[i] = the dispatched row at position i."""
    pieces = []
    for e in range(len(offsets) - 1):
        a, b = int(offsets[e]), int(offsets[e + 1])
        m = (a + b) // 2
        pieces.append((e, a, m))
        pieces.append((e, m, b))
    order = [p for p in reversed(pieces[1::2])] + [p for p in reversed(pieces[0::2])]
    perm, seg_off, seg_exp = [], [0], []
    for e, a, b in order:
        perm.extend(range(a, b))
        seg_off.append(seg_off[-1] + (b - a))
        seg_exp.append(e)
    return np.asarray(perm, np.int64), np.asarray(seg_off, np.int32), np.asarray(seg_exp, np.int32)


@pytest.mark.parametrize("name", list(SEG_CASES))
def test_segments_equal_the_grouped_ffn(name):
    sh = SEG_CASES[name]
    inp = TL.gpu_inputs(sh, seed=3)
    o = TL.run_stages(sh, inp, logits=False)
    assert o["status"] == 0
    dev = inp["x"].device
    offsets = TL.cpu(o["offsets"]).numpy()
    R = int(offsets[-1])
    perm, seg_off, seg_exp = _scrambled(offsets)
    p = torch.as_tensor(perm, device=dev)
    x_rows = o["x_disp"][:R][p].contiguous()
    x_sc = o["x_disp_scales"][:R][p].contiguous() if o["x_disp_scales"] is not None else None
    cfg = M.make_config(T=R, d_model=sh.d_model, n_routed=sh.n_routed, top_k=1, d_ff=sh.d_ff, dtype=sh.dtype)
    ws = torch.empty(M.moe_workspace_size(cfg), dtype=torch.uint8, device=dev)
    M.moe_workspace_init(cfg, ws)
    y = torch.empty((R, sh.d_model), dtype=o["y"].dtype, device=dev)
    g = inp.get
    before = M.moe_kernel_launches()
    M.moe_expert_ffn_segments(cfg, x_rows, x_sc, torch.as_tensor(seg_off, device=dev),
                              torch.as_tensor(seg_exp, device=dev), len(seg_exp), g("W1"), g("W1_scales"),
                              g("b1"), g("W2"), g("W2_scales"), g("b2"), y, ws)
    torch.cuda.synchronize()
    assert M.moe_kernel_launches() - before == 2
    assert M.moe_get_device_status(cfg, ws) == 0
    want = o["y"][:R][p]
    assert torch.equal(y, want), float((y.float() - want.float()).abs().max())


def test_segment_naming_no_expert_is_skipped_and_reported():
    sh = SEG_CASES["bf16"]
    inp = TL.gpu_inputs(sh, seed=4)
    o = TL.run_stages(sh, inp, logits=False)
    dev = inp["x"].device
    offsets = TL.cpu(o["offsets"]).numpy()
    R = int(offsets[-1])
    seg_exp = np.arange(sh.n_routed, dtype=np.int32)
    seg_exp[3] = sh.n_routed                           # names no held expert
    cfg = M.make_config(T=R, d_model=sh.d_model, n_routed=sh.n_routed, top_k=1, d_ff=sh.d_ff, dtype=sh.dtype)
    ws = torch.empty(M.moe_workspace_size(cfg), dtype=torch.uint8, device=dev)
    M.moe_workspace_init(cfg, ws)
    y = torch.full((R, sh.d_model), 7.0, dtype=torch.bfloat16, device=dev)
    g = inp.get
    M.moe_expert_ffn_segments(cfg, o["x_disp"], None, o["offsets"], torch.as_tensor(seg_exp, device=dev),
                              sh.n_routed, g("W1"), None, g("b1"), g("W2"), None, g("b2"), y, ws)
    assert M.moe_get_device_status(cfg, ws) == M.MOE_DEV_BAD_ROUTING
    a, b = int(offsets[3]), int(offsets[4])
    assert bool((y[a:b] == 7.0).all())                 # the skipped segment's rows are untouched
    keep = torch.ones(R, dtype=torch.bool, device=dev)
    keep[a:b] = False
    assert torch.equal(y[keep], o["y"][:R][keep])


EP_CASES = {
    "bf16-shared": MoEShape("e1", 256, 256, 8, 2, 256, n_shared=1, d_ff_shared=128, dtype=DTYPE_BF16),
    "fp8-shared": MoEShape("e2", 128, 256, 16, 4, 256, n_shared=1, d_ff_shared=256, dtype=DTYPE_FP8),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("name", list(EP_CASES))
def test_expert_parallel_one_rank_equals_the_layer(name):
    import torch.distributed as dist
    sh = EP_CASES[name]
    inp = TL.gpu_inputs(sh, seed=6)
    cfg = M.make_config(sh)
    weights = {k: inp.get(k) for k in ("W_r", "logit_bias", "W1", "W1_scales", "b1", "W2", "W2_scales", "b2",
                                       "Ws1", "Ws1_scales", "bs1", "Ws2", "Ws2_scales", "bs2")}
    layer = M.MoELayer(cfg, weights, device=inp["x"].device)
    out, f, P, loss = layer.forward(inp["x"])
    torch.cuda.synchronize()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=inp["x"].device)
    try:
        epl = ep.ExpertParallelMoE(cfg, weights, device=inp["x"].device)
        before = M.moe_kernel_launches()
        eo, ef, eP, eloss = epl.forward(inp["x"])
        torch.cuda.synchronize()
        assert M.moe_kernel_launches() > before
        assert epl.device_status() == 0
        assert torch.equal(eo, out)
        assert torch.equal(epl.topk_idx, layer.topk_idx)
        assert torch.allclose(ef, f, rtol=1e-6, atol=0) and torch.allclose(eP, P, rtol=1e-6, atol=1e-9)
        assert abs(float(eloss) - float(loss)) <= 1e-6 * abs(float(loss))
        del epl
    finally:
        dist.destroy_process_group()

"""GPU parity of every stage and of the whole layer against the CPU oracle,
on seeded inputs small enough for the oracle to finish in seconds but
spanning several tiles, ragged segment tails and the edge cases of the
method (capacity drops, empty experts, K = N_r, one expert, one token)."""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_20_b200 as M
from synthetic import WORKLOADS, DTYPE_BF16, DTYPE_F32, DTYPE_FP8, MoEShape

import moe_testlib as TL

pytestmark = pytest.mark.gpu

CASES = {
    "cfg1-tiny-f32": WORKLOADS[1],
    "f32-ragged-shared-cap": MoEShape("f32r", 203, 128, 6, 2, 192, n_shared=1, d_ff_shared=128,
                                      capacity_factor=1.0, dtype=DTYPE_F32),
    "bf16-ragged-shared-cap": MoEShape("b1", 777, 256, 8, 2, 384, n_shared=1, d_ff_shared=192,
                                       capacity_factor=1.1, dtype=DTYPE_BF16),
    "bf16-fine-grained": MoEShape("b2", 1000, 512, 64, 8, 320, n_shared=2, d_ff_shared=256,
                                  capacity_factor=1.25, dtype=DTYPE_BF16),
    "bf16-nocap": MoEShape("b3", 513, 384, 16, 4, 640, dtype=DTYPE_BF16),
    "bf16-k-equals-n": MoEShape("b4", 100, 128, 4, 4, 128, dtype=DTYPE_BF16),
    "bf16-single-expert": MoEShape("b5", 70, 128, 1, 1, 256, dtype=DTYPE_BF16),
    "bf16-one-token": MoEShape("b6", 1, 256, 8, 2, 256, n_shared=1, d_ff_shared=128, dtype=DTYPE_BF16),
    "f32-generic-router": MoEShape("f32g", 100, 128, 40, 3, 128, dtype=DTYPE_F32),
    "bf16-e24-small-router": MoEShape("b7", 300, 256, 24, 3, 256, dtype=DTYPE_BF16),
    "bf16-e128-tc-router": MoEShape("b8", 600, 256, 128, 4, 128, n_shared=1, d_ff_shared=128,
                                    dtype=DTYPE_BF16),
    # tensor-core router on CTA pairs with a 128-wide expert tile (nine token
    # tiles: the last pair has one), and 8 experts too wide for the
    # shared-memory router (d = 5632): a 32-wide tile with zero rows past N_r
    "bf16-e128-pair-router": MoEShape("b9", 1100, 256, 128, 4, 128, dtype=DTYPE_BF16),
    "bf16-e8-wide-tc-router": MoEShape("b10", 300, 5632, 8, 2, 128, dtype=DTYPE_BF16),
    "fp8-ragged-shared": MoEShape("f1", 300, 512, 16, 4, 256, n_shared=1, d_ff_shared=384, dtype=DTYPE_FP8),
    "fp8-decode-skewed": MoEShape("f2", 37, 1024, 256, 8, 256, n_shared=1, d_ff_shared=256,
                                  dtype=DTYPE_FP8, zipf_logit_bias=True),
    # selection-only bias on each router path: small (N_r <= 32), tensor-core, fp32 generic
    "bf16-selbias-small-router": MoEShape("s1", 300, 256, 8, 2, 256, dtype=DTYPE_BF16,
                                          bias_mode=1, selection_bias=True),
    "bf16-selbias-tc-router": MoEShape("s2", 600, 256, 128, 4, 128, n_shared=1, d_ff_shared=128,
                                       capacity_factor=1.0, dtype=DTYPE_BF16, bias_mode=1, selection_bias=True),
    "f32-selbias-generic-router": MoEShape("s3", 100, 128, 40, 3, 128, dtype=DTYPE_F32,
                                           bias_mode=1, selection_bias=True),
    "fp8-selbias": MoEShape("s4", 200, 512, 64, 8, 256, n_shared=1, d_ff_shared=128,
                            dtype=DTYPE_FP8, bias_mode=1, selection_bias=True),
    # limits of the interface: top-16 of 256 experts, 8 shared experts, one FP8 token
    "bf16-k16-e256": MoEShape("m1", 200, 256, 256, 16, 128, dtype=DTYPE_BF16),
    "bf16-8-shared": MoEShape("m2", 96, 128, 8, 2, 128, n_shared=8, d_ff_shared=64, dtype=DTYPE_BF16),
    "fp8-one-token": MoEShape("m3", 1, 256, 16, 4, 256, n_shared=1, d_ff_shared=128, dtype=DTYPE_FP8),
    # d_model not a multiple of 128 (bf16 and fp32 take multiples of 64): a
    # K tail in the first layer and the router, an N tail of 64 columns in
    # the second, rows of 640 / 384 bytes in the dispatch copy and combine;
    # on the small, tensor-core and generic routers
    "bf16-d320-shared-cap": MoEShape("t1", 333, 320, 8, 2, 192, n_shared=1, d_ff_shared=128,
                                     capacity_factor=1.1, dtype=DTYPE_BF16),
    "bf16-d192-tc-router": MoEShape("t2", 300, 192, 64, 4, 256, dtype=DTYPE_BF16),
    "f32-d192-generic-router": MoEShape("t3", 150, 192, 40, 2, 192, dtype=DTYPE_F32),
    # top-1 routing over many experts (one slot per token), with a capacity
    # that drops and with FP8
    "bf16-top1-cap": MoEShape("u1", 500, 256, 16, 1, 256, capacity_factor=1.0, dtype=DTYPE_BF16),
    "fp8-top1-shared": MoEShape("u2", 300, 512, 32, 1, 256, n_shared=1, d_ff_shared=256, dtype=DTYPE_FP8),
    # capacity variants: slot-major priority, overflow pass-through, both
    "bf16-slotmajor-cap": MoEShape("c1", 300, 256, 8, 2, 256, capacity_factor=0.8, dtype=DTYPE_BF16,
                                   capacity_priority=1),
    "bf16-passthrough-cap": MoEShape("c2", 300, 256, 8, 2, 256, capacity_factor=0.8, dtype=DTYPE_BF16,
                                     overflow_mode=1),
    "f32-slotmajor-passthrough": MoEShape("c3", 203, 128, 6, 2, 192, n_shared=1, d_ff_shared=128,
                                          capacity_factor=0.75, dtype=DTYPE_F32, capacity_priority=1,
                                          overflow_mode=1),
    "fp8-slotmajor-passthrough": MoEShape("c4", 300, 512, 16, 4, 256, n_shared=1, d_ff_shared=128,
                                          capacity_factor=0.75, dtype=DTYPE_FP8, capacity_priority=1,
                                          overflow_mode=1),
}


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name", list(CASES))
def test_stage_and_layer_parity(name):
    require_gpu()
    sh = CASES[name]
    inp = TL.gpu_inputs(sh, seed=1234)
    n0 = M.moe_kernel_launches()
    o = TL.run_stages(sh, inp)
    n_stages = M.moe_kernel_launches() - n0
    assert o["status"] == 0
    rt_prod = TL.check_routing(sh, inp, o)
    TL.check_dispatch(sh, inp, o, rt_prod)
    TL.check_expert_ffn(sh, inp, o, rt_prod)
    TL.check_combine(sh, o, rt_prod, x=inp["x"])
    n1 = M.moe_kernel_launches()
    lay = TL.run_layer(sh, inp)
    n_layer = M.moe_kernel_launches() - n1
    assert lay["status"] == 0
    # stages: router >= 1, dispatch 3, two grouped GEMMs, combine, balance;
    # the fused entry point computes the balance statistics in the dispatch scan
    assert n_layer == n_stages - 1 and n_stages >= 8, (n_layer, n_stages)
    # the fused entry point runs the same kernels in the same order
    assert torch.equal(lay["out"], o["out"])
    assert torch.equal(lay["topk_idx"], o["topk_idx"])
    assert torch.equal(lay["P"], o["P"]) and torch.equal(lay["f"], o["f"])
    err, excluded = TL.check_end_to_end(sh, inp, lay["out"], TL.cpu(lay["topk_idx"]).numpy())
    assert excluded <= max(2, sh.T // 100)
    assert err < TL.TOL_REL_FROB[sh.dtype], err


def test_all_tokens_to_one_expert_with_capacity():
    require_gpu()
    sh = MoEShape("hot", 500, 256, 8, 2, 256, capacity_factor=1.0, dtype=DTYPE_BF16)
    inp = TL.gpu_inputs(sh, seed=7)
    bias = torch.zeros(8, device="cuda")
    bias[3] = 60.0                        # every token's first choice is expert 3
    bias[5] = -60.0                       # expert 5 is never chosen (empty segment)
    inp["logit_bias"] = bias
    o = TL.run_stages(sh, inp)
    rt = TL.check_routing(sh, inp, o)
    C = rt["C"]
    assert rt["plan"]["counts"][3] == 500 and rt["plan"]["kept"][3] == C
    assert rt["plan"]["counts"][5] == 0
    TL.check_dispatch(sh, inp, o, rt)
    TL.check_expert_ffn(sh, inp, o, rt)
    TL.check_combine(sh, o, rt, x=inp["x"])
    err, _ = TL.check_end_to_end(sh, inp, o["out"], TL.cpu(o["topk_idx"]).numpy())
    assert err < TL.TOL_REL_FROB[sh.dtype]


def test_bad_routing_is_flagged_and_dropped():
    require_gpu()
    sh = MoEShape("bad", 64, 128, 8, 2, 128, dtype=DTYPE_BF16)
    inp = TL.gpu_inputs(sh, seed=3)
    cfg = M.make_config(sh)
    dev = "cuda"
    idx = torch.tensor(np.stack([np.arange(64) % 8, (np.arange(64) + 1) % 8], 1), dtype=torch.int32, device=dev)
    idx[5, 1] = 8                         # out of range
    idx[9, 1] = idx[9, 0]                 # repeated within the token
    ws = torch.empty(M.moe_workspace_size(cfg), dtype=torch.uint8, device=dev)
    M.moe_workspace_init(cfg, ws)
    E, T, K = 8, 64, 2
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    kept = torch.empty_like(counts)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    slot_row = torch.empty((T, K), dtype=torch.int32, device=dev)
    row_slot = torch.empty(T * K, dtype=torch.int32, device=dev)
    x_disp = torch.empty((T * K, 128), dtype=torch.bfloat16, device=dev)
    M.moe_dispatch(cfg, inp["x"], idx, counts, kept, offsets, slot_row, row_slot, x_disp, None, ws)
    status = M.moe_get_device_status(cfg, ws, clear=True)
    assert status & M.MOE_DEV_BAD_ROUTING
    sr = slot_row.cpu().numpy()
    assert sr[5, 1] == -2 and sr[9, 1] == -2        # invalid index (-1 means over the capacity)
    assert int(counts.sum()) == T * K - 2
    assert M.moe_get_device_status(cfg, ws) == 0


def test_bounded_wait_reports_timeout_and_context_survives():
    require_gpu()
    sh = MoEShape("to", 64, 128, 8, 2, 128, dtype=DTYPE_BF16)
    cfg = M.make_config(sh)
    ws = torch.empty(M.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(cfg, ws)
    M.moe_selftest_wait_timeout(cfg, 20_000_000, ws)          # 20 ms
    assert M.moe_get_device_status(cfg, ws, clear=True) & M.MOE_DEV_TIMEOUT
    inp = TL.gpu_inputs(sh, seed=5)
    o = TL.run_stages(sh, inp)                                  # the context still works
    assert o["status"] == 0
    TL.check_routing(sh, inp, o)


def test_layer_is_deterministic():
    require_gpu()
    sh = CASES["bf16-fine-grained"]
    inp = TL.gpu_inputs(sh, seed=99)
    a = TL.run_layer(sh, inp)
    b = TL.run_layer(sh, inp)
    assert torch.equal(a["out"], b["out"]) and torch.equal(a["P"], b["P"]) and torch.equal(a["loss"], b["loss"])


def test_host_batches_pipeline_matches_forward():
    """MoELayer.forward_host_batches (copies on their own streams, double
    buffers) returns, for every batch, exactly what forward() returns."""
    require_gpu()
    sh = CASES["bf16-ragged-shared-cap"]
    inp = TL.gpu_inputs(sh, seed=7)
    layer = M.MoELayer(M.make_config(sh), inp, device=inp["x"].device)
    gen = torch.Generator().manual_seed(11)
    xs = [torch.randn(sh.T, sh.d_model, generator=gen).to(torch.bfloat16).pin_memory() for _ in range(5)]
    outs = [torch.empty(sh.T, sh.d_model, dtype=torch.bfloat16).pin_memory() for _ in range(5)]
    losses = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(5)]
    layer.forward_host_batches(xs, outs, losses)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    for k in range(5):
        out, _, _, loss = layer.forward(xs[k].to(inp["x"].device))
        torch.cuda.synchronize()
        assert torch.equal(outs[k], out.cpu()), k
        assert torch.equal(losses[k], loss.cpu()), k


def test_fp8_tiny_block_scale_stays_normal():
    """A 128-column block whose largest magnitude is below 448 * 2^-126 gets
    the scale 2^-126, on the GPU as in the oracle, so codes and scales of the
    dispatched rows still match bit for bit and the layer output stays within
    tolerance."""
    require_gpu()
    sh = MoEShape("tiny-amax", 200, 512, 16, 4, 256, n_shared=1, d_ff_shared=128, dtype=DTYPE_FP8)
    inp = TL.gpu_inputs(sh, seed=21)
    x = inp["x"].clone()
    x[3, 128:256] = (x[3, 128:256].float() * 1e-37).to(torch.bfloat16)     # amax ~ 3e-37
    x[50, 0:128] = 1e-38                                                   # below 2^-126
    x[77, 384:512] = (x[77, 384:512].float() * 2.0 ** -130).to(torch.bfloat16)
    inp["x"] = x
    o = TL.run_stages(sh, inp)
    assert o["status"] == 0
    rt_prod = TL.check_routing(sh, inp, o)
    TL.check_dispatch(sh, inp, o, rt_prod)
    sc = TL.cpu(o["x_disp_scales"]).double().numpy()
    rc = o["r_cap"]
    assert sc[rc + 3, 1] == 2.0 ** -126 and sc[rc + 50, 0] == 2.0 ** -126 and sc[rc + 77, 3] == 2.0 ** -126
    TL.check_expert_ffn(sh, inp, o, rt_prod)
    err, _ = TL.check_end_to_end(sh, inp, o["out"], TL.cpu(o["topk_idx"]).numpy())
    assert err < TL.TOL_REL_FROB[sh.dtype], err

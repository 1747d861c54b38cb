"""moe_dispatch_noalloc: dispatch for callers that cannot allocate device
memory (for example a plugin inside a host framework that owns every device
allocation).  Its scratch lives in a fixed 2 MiB device array of the library
instead of a caller workspace.

Calls in a row, through the C ABI, must give exactly what moe_dispatch gives
on the same inputs and exactly what the oracle's dispatch plan and FP8
quantiser give on the same routing; each call runs on whatever the previous
one left in the shared array.  The cases cover token-order and slot-major
capacity priority (one bitmap plane per slot), the last size that fits the
array, and the first that does not.  This file is collected last so that a
failure here leaves every other test already run."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_20_b200 as M
from synthetic import DTYPE_BF16, DTYPE_FP8, MoEShape

import moe_testlib as TL

# token order, FP8 with a shared expert (the quantised copy of every token)
FP8_SHARED = MoEShape("na1", 1500, 512, 64, 8, 256, n_shared=1, d_ff_shared=256, dtype=DTYPE_FP8)
# token order with a capacity limit
BF16_CAP = MoEShape("na2", 777, 256, 16, 4, 256, capacity_factor=1.1, dtype=DTYPE_BF16)
# slot-major priority: K bitmap planes; 2 * 8 * (16384 / 32) * 64 * 4 bytes = 2 MiB, the array's size
SLOT_MAJOR_EDGE = MoEShape("na3", 16384, 128, 64, 8, 128, capacity_factor=1.0, dtype=DTYPE_BF16,
                           capacity_priority=1)


def _outputs(sh, dev):
    cfg = M.make_config(sh)
    cap, r_cap, x_rows, _ = M.moe_buffer_rows(cfg)
    fp8 = sh.dtype == DTYPE_FP8
    i32 = dict(dtype=torch.int32, device=dev)
    return {
        "counts": torch.full((sh.n_routed,), -7, **i32),
        "kept": torch.full((sh.n_routed,), -7, **i32),
        "offsets": torch.full((sh.n_routed + 1,), -7, **i32),
        "slot_row": torch.full((sh.T, sh.top_k), -7, **i32),
        "row_slot": torch.full((max(r_cap, 1),), -7, **i32),
        "x_disp": torch.zeros((x_rows, sh.d_model), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev),
        "x_disp_scales": torch.zeros((x_rows, sh.d_model // 128), dtype=torch.float32, device=dev) if fp8 else None,
    }


def _dispatch_both(sh, seed):
    dev = "cuda"
    inp = TL.gpu_inputs(sh, seed=seed, device=dev)
    cfg = M.make_config(sh)
    ws = torch.empty(M.moe_workspace_size(cfg), dtype=torch.uint8, device=dev)
    M.moe_workspace_init(cfg, ws)
    idx = torch.empty((sh.T, sh.top_k), dtype=torch.int32, device=dev)
    gates = torch.empty((sh.T, sh.top_k), dtype=torch.float32, device=dev)
    M.moe_route(cfg, inp["x"], inp["W_r"], inp["logit_bias"], idx, gates, None, ws)
    ref = _outputs(sh, dev)
    M.moe_dispatch(cfg, inp["x"], idx, ref["counts"], ref["kept"], ref["offsets"], ref["slot_row"],
                   ref["row_slot"], ref["x_disp"], ref["x_disp_scales"], ws)
    got = _outputs(sh, dev)
    n0 = M.moe_kernel_launches()
    M.moe_dispatch_noalloc(cfg, inp["x"], idx, got["counts"], got["kept"], got["offsets"], got["slot_row"],
                           got["row_slot"], got["x_disp"], got["x_disp_scales"])
    assert M.moe_kernel_launches() - n0 == 3          # bitmap, scan, scatter: the same kernels
    torch.cuda.synchronize()
    return inp, idx, ref, got


def _check_against_oracle(sh, inp, idx, got):
    """The oracle's plan on the product's own routing, and its quantiser."""
    cap, r_cap, _, _ = M.moe_buffer_rows(M.make_config(sh))
    C = O.capacity_of(sh.T, sh.top_k, sh.n_routed, sh.capacity_factor)
    assert (C if C is not None else -1) == cap
    plan = O.dispatch_plan(TL.cpu(idx).numpy(), sh.n_routed, C,
                           "slot" if sh.capacity_priority == 1 else "token")
    o = dict(got, r_cap=r_cap)
    TL.check_dispatch(sh, inp, o, {"plan": plan})


@pytest.mark.gpu
def test_dispatch_noalloc_matches_dispatch_and_oracle_on_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    for sh, seed in ((FP8_SHARED, 11), (BF16_CAP, 12), (SLOT_MAJOR_EDGE, 13), (BF16_CAP, 14)):
        inp, idx, ref, got = _dispatch_both(sh, seed)
        for k in ref:
            if ref[k] is None:
                assert got[k] is None
                continue
            # dispatch is integer / byte work: bit-exact, as in the other dispatch tests
            assert torch.equal(ref[k], got[k]), (sh.name, k)
        _check_against_oracle(sh, inp, idx, got)


def _rejected(sh):
    cfg = M.make_config(sh)
    p = 0x100000                      # never dereferenced: the size check comes first
    L = M.lib()
    n0 = M.moe_kernel_launches()
    st = L.moe_dispatch_noalloc(ctypes.byref(cfg), p, p, p, p, p, p, p, p,
                                p if sh.dtype == DTYPE_FP8 else None, None)
    assert M.moe_kernel_launches() == n0, "a rejected call launched a kernel"
    return st


def test_dispatch_noalloc_rejects_sizes_beyond_its_scratch():
    # token order: 2 * ceil(T/32) * N_r * 4 bytes > 2 MiB
    assert _rejected(MoEShape("too-big", 40000, 128, 256, 8, 128, dtype=DTYPE_BF16)) == M.MOE_ERR_UNSUPPORTED
    # one more 32-token word than the slot-major edge case above
    over = SLOT_MAJOR_EDGE.replace(name="over", T=SLOT_MAJOR_EDGE.T + 1)
    assert _rejected(over) == M.MOE_ERR_UNSUPPORTED
    # FP8 without its scale output is an argument error, also before any launch
    fp8 = FP8_SHARED.replace(name="noscales")
    cfg = M.make_config(fp8)
    p = 0x100000
    n0 = M.moe_kernel_launches()
    assert M.lib().moe_dispatch_noalloc(ctypes.byref(cfg), p, p, p, p, p, p, p, p, None, None) == \
        M.MOE_ERR_INVALID_ARG
    assert M.moe_kernel_launches() == n0

"""moe_dispatch_noalloc: dispatch for callers that cannot allocate device
memory (for example a plugin inside a host framework that owns every device
allocation).  Its scratch lives in a fixed 2 MiB device array of the library
instead of a caller workspace.  Two calls in a row, through the C ABI, must
give exactly what moe_dispatch gives on the same inputs; the second call runs
on whatever the first one left in the shared array.  This file is collected
last so that a failure here leaves every other test already run."""
import pytest
import torch

import sparse_mixture_experts_20_b200 as M
from synthetic import DTYPE_BF16, DTYPE_FP8, MoEShape

import moe_testlib as TL

pytestmark = pytest.mark.gpu


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
    M.moe_dispatch_noalloc(cfg, inp["x"], idx, got["counts"], got["kept"], got["offsets"], got["slot_row"],
                           got["row_slot"], got["x_disp"], got["x_disp_scales"])
    torch.cuda.synchronize()
    return ref, got


def test_dispatch_noalloc_matches_dispatch_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    first = MoEShape("na1", 1500, 512, 64, 8, 256, n_shared=1, d_ff_shared=256, dtype=DTYPE_FP8)
    second = MoEShape("na2", 777, 256, 16, 4, 256, capacity_factor=1.1, dtype=DTYPE_BF16)
    for sh, seed in ((first, 11), (second, 12)):
        ref, got = _dispatch_both(sh, seed)
        for k in ref:
            if ref[k] is None:
                assert got[k] is None
                continue
            # dispatch is integer / byte work: bit-exact, as in the other dispatch tests
            assert torch.equal(ref[k], got[k]), (sh.name, k)


def test_dispatch_noalloc_rejects_sizes_beyond_its_scratch():
    # 2 * ceil(T/32) * N_r * 4 bytes > 2 MiB
    sh = MoEShape("too-big", 40000, 128, 256, 8, 128, dtype=DTYPE_BF16)
    cfg = M.make_config(sh)
    p = 0x100000
    L = M.lib()
    import ctypes
    st = L.moe_dispatch_noalloc(ctypes.byref(cfg), p, p, p, p, p, p, p, p, None, None)
    assert st == M.MOE_ERR_UNSUPPORTED

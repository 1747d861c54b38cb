"""FP8 block scales that differ from block to block ("DeepSeek DeepEP"
§DeepEP とは: activations with one scale per 1x128 block, weights with one
per 128x128 block).

Seeded N(0,1) activations quantise to nearly the same power-of-two scale in
every 128-column block, and N(0, 1/fan_in) weights likewise, so a scale taken
from the wrong k-block or weight block would mostly go unnoticed by the other
FP8 cases.  Here every 128-column block of x is multiplied by its own power
of two (1/8 .. 8) and every weight block's scale by its own power of two
(1/4 .. 4).  Both changes are exact (the codes are unchanged and the scales
stay powers of two, which UE8M0 represents) and are seen identically by the
kernels and the oracle.  Stage and end-to-end parity as in test_gpu_parity,
for a layer whose every K is a multiple of 512 (the scale writers read four
k-blocks of scales at a time) and one where none is (one k-block at a
time)."""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_20_b200 as M
from synthetic import DTYPE_FP8, MoEShape, make_inputs

import moe_testlib as TL

CASES = {
    "k-multiple-of-512": MoEShape("fs1", 260, 1024, 8, 2, 512, n_shared=1, d_ff_shared=512, dtype=DTYPE_FP8),
    "k-not-multiple-of-512": MoEShape("fs2", 260, 640, 8, 2, 384, n_shared=1, d_ff_shared=256,
                                      dtype=DTYPE_FP8),
}


def _vary_scales(sh, inp):
    x = inp["x"]
    nb = sh.d_model // 128
    f = torch.tensor([2.0 ** ((3 * j) % 7 - 3) for j in range(nb)], device=x.device)
    inp["x"] = (x.float().view(sh.T, nb, 128) * f.view(1, nb, 1)).view(sh.T, sh.d_model).to(x.dtype).contiguous()
    assert torch.equal(inp["x"].float().view(sh.T, nb, 128) / f.view(1, nb, 1), x.float().view(sh.T, nb, 128))
    for key in ("W1_scales", "W2_scales", "Ws1_scales", "Ws2_scales"):
        s = inp.get(key)
        if s is None:
            continue
        idx = torch.arange(s.numel(), device=s.device).view(s.shape)
        inp[key] = (s * torch.pow(2.0, ((idx * 7) % 5 - 2).to(s.dtype))).contiguous()
    return inp


def test_a_misplaced_scale_is_visible_here_and_not_with_plain_inputs():
    """On the CPU, with the oracle: the first expert's output with each W1
    block scale taken from the neighbouring k-block differs by far more than
    the FP8 tolerance on these inputs, and not at all on the plain seeded
    inputs (whose weight block scales are all equal)."""
    sh = CASES["k-multiple-of-512"]

    def planted_error(inp):
        W1, b1, W2, b2 = O.expert_weights(inp, "W", 0, True)
        x = O.to_f64(inp["x"][:64])
        ref = O.expert_ffn(x, W1, b1, W2, b2, fp8_hidden=True)
        bad = dict(inp, W1_scales=torch.roll(inp["W1_scales"], 1, dims=-1))
        W1b = O.expert_weights(bad, "W", 0, True)[0]
        return np.linalg.norm(O.expert_ffn(x, W1b, b1, W2, b2, fp8_hidden=True) - ref) / np.linalg.norm(ref)

    plain = make_inputs(sh, 77, device="cpu")
    assert planted_error(_vary_scales(sh, dict(plain))) > 10 * TL.TOL_REL_FROB[sh.dtype]
    assert planted_error(plain) < TL.TOL_REL_FROB[sh.dtype]


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_varied_block_scales(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sh = CASES[name]
    inp = _vary_scales(sh, TL.gpu_inputs(sh, seed=77))
    # the activation scales of the dispatched rows really differ along K
    o = TL.run_stages(sh, inp)
    assert o["status"] == 0
    xs = o["x_disp_scales"][: int(TL.cpu(o["offsets"])[-1])]
    assert xs.numel() > 0 and bool((xs != xs[:, :1]).any())
    rt_prod = TL.check_routing(sh, inp, o)
    TL.check_dispatch(sh, inp, o, rt_prod)
    TL.check_expert_ffn(sh, inp, o, rt_prod)
    TL.check_combine(sh, o, rt_prod, x=inp["x"])
    lay = TL.run_layer(sh, inp)
    assert lay["status"] == 0
    assert torch.equal(lay["out"], o["out"])
    err, excluded = TL.check_end_to_end(sh, inp, lay["out"], TL.cpu(lay["topk_idx"]).numpy())
    assert excluded <= max(2, sh.T // 100)
    assert err < TL.TOL_REL_FROB[sh.dtype], err
    assert M.moe_kernel_launches() > 0

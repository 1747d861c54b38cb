"""The synthetic input generator follows its stated recipe (CPU only):
x ~ N(0, 1) in the activation dtype; W_r, W1 ~ N(0, 1/d_model), W2 ~
N(0, 1/d_ff); biases ~ N(0, 0.01) (std 0.1) in fp32; the decode workload's
Zipf bias 1.5 ln(1/rank) over a permutation of ranks 1..N_r; the
selection-only bias ~ N(0, 0.25); FP8 weights encoded per 128x128 block with
the smallest power-of-two scale that brings the block's amax to <= 448; and
every draw fixed by the seed."""
import math
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from synthetic import WORKLOADS, DTYPE_BF16, DTYPE_F32, DTYPE_FP8, MoEShape, encode_fp8_blocks, make_inputs  # noqa: E402

SH = MoEShape("recipe", 512, 256, 8, 2, 512, n_shared=1, d_ff_shared=256, dtype=DTYPE_BF16)


def _std_ok(t, want, rel=0.03):
    v = t.double()
    return abs(float(v.mean())) < 4 * want / math.sqrt(v.numel()) + 1e-12 and abs(float(v.std()) / want - 1) < rel


def test_distributions_and_dtypes():
    inp = make_inputs(SH, seed=3)
    d, f = SH.d_model, SH.d_ff
    assert inp["x"].dtype == torch.bfloat16 and inp["W1"].dtype == torch.bfloat16
    assert inp["W_r"].dtype == torch.float32 and inp["b1"].dtype == torch.float32
    assert _std_ok(inp["x"], 1.0)
    assert _std_ok(inp["W_r"], 1 / math.sqrt(d))
    assert _std_ok(inp["W1"], 1 / math.sqrt(d)) and _std_ok(inp["Ws1"], 1 / math.sqrt(d))
    assert _std_ok(inp["W2"], 1 / math.sqrt(f)) and _std_ok(inp["Ws2"], 1 / math.sqrt(SH.d_ff_shared))
    for b in ("b1", "b2", "bs1", "bs2"):
        assert _std_ok(inp[b], 0.1, rel=0.08), b
    assert inp["logit_bias"] is None
    assert inp["W1"].shape == (SH.n_routed, f, d) and inp["W2"].shape == (SH.n_routed, d, f)
    assert inp["Ws1"].shape == (1, SH.d_ff_shared, d) and inp["Ws2"].shape == (1, d, SH.d_ff_shared)
    f32 = make_inputs(SH.replace(dtype=DTYPE_F32), seed=3, route_only=True)
    assert f32["x"].dtype == torch.float32 and "W1" not in f32


def test_seed_fixes_every_draw():
    a, b = make_inputs(SH, seed=5), make_inputs(SH, seed=5)
    c = make_inputs(SH, seed=6)
    for k, v in a.items():
        if v is not None:
            assert torch.equal(v, b[k]), k
    assert not torch.equal(a["x"], c["x"]) and not torch.equal(a["W1"], c["W1"])


def test_zipf_logit_bias_of_the_decode_workload():
    sh = WORKLOADS[5]
    b = make_inputs(sh.replace(T=4), seed=0, route_only=True)["logit_bias"].double().numpy()
    ranks = np.exp(-b / 1.5)                       # b = 1.5 ln(1/rank)
    assert np.allclose(ranks, np.round(ranks), rtol=0, atol=1e-3)
    assert sorted(np.round(ranks).astype(int)) == list(range(1, sh.n_routed + 1))
    assert b.max() == 0.0 and np.isclose(b.min(), -1.5 * math.log(sh.n_routed), atol=1e-5)


def test_selection_bias_draw():
    sh = MoEShape("sb", 4, 128, 256, 8, 128, selection_bias=True, bias_mode=1)
    b = make_inputs(sh, seed=1, route_only=True)["logit_bias"]
    assert b.shape == (256,) and abs(float(b.std()) / 0.5 - 1) < 0.15


@pytest.mark.parametrize("std", [1e-3, 0.02, 3.0])
def test_fp8_block_encoding(std):
    g = torch.Generator().manual_seed(11)
    w = torch.empty((256, 384)).normal_(0.0, std, generator=g)
    w[128:, :128] = 0.0                                      # an all-zero block
    codes, scales = encode_fp8_blocks(w)
    assert codes.dtype == torch.uint8 and scales.shape == (2, 3)
    mant, _ = torch.frexp(scales.double())
    assert torch.all(mant == 0.5)                            # powers of two
    assert scales[1, 0] == 1.0
    vals = codes.view(torch.float8_e4m3fn).float()
    for i in range(2):
        for j in range(3):
            blk = w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            amax = float(blk.abs().max())
            if amax == 0.0:
                continue
            s = float(scales[i, j])
            assert amax / s <= 448.0 < 2 * amax / s             # the smallest such power of two
            q = vals[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            assert float(q.abs().max()) <= 448.0
            # round to nearest: within half an e4m3 step (2^-4 relative) or the subnormal step
            err = (q * s - blk).abs()
            assert torch.all(err <= torch.maximum(blk.abs() * 2.0 ** -4, torch.tensor(2.0 ** -10 * s)))


def test_fp8_workload_weights_are_encoded_blocks():
    sh = MoEShape("f8", 8, 256, 2, 2, 256, n_shared=1, d_ff_shared=128, dtype=DTYPE_FP8)
    inp = make_inputs(sh, seed=2)
    assert inp["W1"].dtype == torch.uint8 and inp["W1_scales"].shape == (2, 2, 2)
    assert inp["Ws2"].dtype == torch.uint8 and inp["Ws2_scales"].shape == (1, 2, 1)
    assert inp["x"].dtype == torch.bfloat16

"""Exact ties in the router on the GPU ("Sparse MoE Top-Kルーティング"
§ルーティングの仕組み; ties go to the lower expert index).

The router-weight rows of a set Z of experts are zero and their logit bias is
0, so every token's logits over Z are exactly +0 (a signed zero from the
products plus +0); every other expert gets a bias of -50 and is never
chosen.  Top-K must then be the K lowest indices of Z in ascending order,
with equal gates 1/K -- on the small router (N_r = 8) and the tensor-core
router (N_r = 64)."""
import numpy as np
import pytest
import torch

import moe_testlib as TL
from synthetic import DTYPE_BF16, DTYPE_F32, MoEShape

pytestmark = pytest.mark.gpu

CASES = {
    "small-router-bf16": (MoEShape("tie1", 96, 128, 8, 4, 128, dtype=DTYPE_BF16), [1, 2, 4, 5, 7]),
    "small-router-f32": (MoEShape("tie2", 64, 128, 8, 2, 128, dtype=DTYPE_F32), [3, 6, 7]),
    "tc-router-bf16": (MoEShape("tie3", 160, 128, 64, 8, 128, dtype=DTYPE_BF16),
                       [2, 9, 10, 17, 33, 40, 41, 50, 51, 63]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_exact_ties_go_to_the_lower_index(name):
    sh, Z = CASES[name]
    inp = TL.gpu_inputs(sh, seed=21)
    W_r = inp["W_r"].clone()
    W_r[Z] = 0.0
    inp["W_r"] = W_r
    bias = torch.full((sh.n_routed,), -50.0, device=W_r.device)
    bias[Z] = 0.0
    inp["logit_bias"] = bias
    o = TL.run_stages(sh, inp)
    assert o["status"] == 0
    logits = TL.cpu(o["logits"]).numpy()
    assert np.all(logits[:, Z] == 0.0)                  # the ties are exact
    idx = TL.cpu(o["topk_idx"]).numpy()
    want = np.array(sorted(Z)[:sh.top_k], dtype=np.int32)
    assert np.array_equal(idx, np.tile(want, (sh.T, 1)))
    g = TL.cpu(o["gates"]).numpy()
    assert np.allclose(g, 1.0 / sh.top_k, rtol=0, atol=1e-6)
    rt = TL.check_routing(sh, inp, o)                  # and the oracle agrees on these logits
    TL.check_dispatch(sh, inp, o, rt)

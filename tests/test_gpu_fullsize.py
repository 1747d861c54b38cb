"""GPU parity at the full sizes of the four named large workloads, in the
launch configuration the benchmark times (moe_layer_forward).  Routing,
counts, offsets and the permutation are checked for every token; expert
outputs and the layer output on a seeded sample of rows / tokens that the
oracle computes one by one."""
import numpy as np
import pytest
import torch

import oracle as O
from synthetic import WORKLOADS

import moe_testlib as TL

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cid", [2, 3, 4, 5])
def test_fullsize_config(cid):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sh = WORKLOADS[cid]
    inp = TL.gpu_inputs(sh, seed=0, on_device_gen=True)
    o = TL.run_stages(sh, inp)
    assert o["status"] == 0
    rt_prod = TL.check_routing(sh, inp, o)
    TL.check_dispatch(sh, inp, o, rt_prod)
    rng = np.random.default_rng(cid)
    R = rt_prod["plan"]["R"]
    rows = np.sort(rng.choice(R, size=min(R, 96), replace=False))
    toks = np.sort(rng.choice(sh.T, size=min(sh.T, 32), replace=False))
    TL.check_expert_ffn(sh, inp, o, rt_prod, rows=rows, tokens=toks)
    lay = TL.run_layer(sh, inp)
    assert lay["status"] == 0
    assert torch.equal(lay["out"], o["out"])
    rt = O.route(sh, inp)
    err, excluded = TL.check_end_to_end(sh, inp, lay["out"], TL.cpu(lay["topk_idx"]).numpy(),
                                        tokens=toks, routing=rt)
    print(f"cfg{cid}: rel_frob={err:.3e} excluded={excluded} max_load={rt_prod['plan']['counts'].max()} "
          f"touched={(rt_prod['plan']['counts'] > 0).sum()} drops={int(rt_prod['plan']['counts'].sum() - R)}")
    assert err < TL.TOL_REL_FROB[sh.dtype], err

"""GPU parity at the full sizes of the four named large workloads, in the
launch configuration the benchmark times (moe_layer_forward).  Routing,
counts, offsets and the permutation are checked for every token; expert
outputs and the layer output on a sample of rows / tokens that the oracle
computes one by one: seeded random rows plus, for every expert segment, its
first and last rows and the first row of its last 128-row tile and of its
last 256-row tile pair (the ragged tails of the grouped GEMMs), and the
first, last and last-tile tokens of the shared experts.  Each sampled row
must meet the per-row bound as well as the whole-sample one."""
import numpy as np
import pytest
import torch

import oracle as O
from synthetic import WORKLOADS

import moe_testlib as TL


def segment_edge_rows(offsets):
    """First and last row of every non-empty segment, and the first row of its
    last 128-row m-tile and of its last 256-row pair of m-tiles."""
    out = []
    for e in range(len(offsets) - 1):
        o0, o1 = int(offsets[e]), int(offsets[e + 1])
        n = o1 - o0
        if n <= 0:
            continue
        out += [o0, o1 - 1, o0 + 128 * ((n - 1) // 128), o0 + 256 * ((n - 1) // 256)]
    return np.unique(np.asarray(out, np.int64))


def test_segment_edge_rows_cover_the_tails():
    rows = segment_edge_rows(np.array([0, 300, 300, 301, 1000]))
    # segment 0: 300 rows -> 0, 299, 256 (last 128-tile and last pair start at 256)
    # segment 1 is empty; segment 2: one row (300); segment 3: rows 301..999
    # (699 rows: last 128-tile at 301 + 640, last pair at 301 + 512)
    assert list(rows) == [0, 256, 299, 300, 301, 813, 941, 999]


@pytest.mark.gpu
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
    rows = np.union1d(rows, segment_edge_rows(rt_prod["plan"]["offsets"]))
    toks = np.sort(rng.choice(sh.T, size=min(sh.T, 32), replace=False))
    toks = np.union1d(toks, [0, sh.T - 1, 128 * ((sh.T - 1) // 128), 256 * ((sh.T - 1) // 256)])
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

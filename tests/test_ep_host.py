"""Expert parallelism, host side, on CPU ("エキスパート並列（Expert
Parallelism）" §推論フロー): the plan of sparse_mixture_experts_20_b200.ep (which
rows go to which rank, the received segments) and its all_to_all exchange, on
two and four gloo ranks.  The layer arithmetic on each rank is the oracle's
(the CUDA kernels need a GPU): every rank routes its own tokens, dispatches
them in expert order, sends each expert owner its rows, the owners run their
experts on the received segments, the outputs come back and each rank
combines.  The result must be the single-process oracle layer on the same
tokens, and the balance statistics those of all ranks' tokens together."""
import datetime
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from sparse_mixture_experts_20_b200 import ep  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_plan_by_hand():
    # 2 ranks, 4 experts (2 each): this rank's dispatched rows per expert
    assert ep.send_splits([3, 0, 2, 5], 2) == [3, 7]
    assert ep.expert_range(1, 2, 4) == (2, 4)
    # received: from source 0 (1, 2) rows for held experts (0, 1), from source 1 (0, 4)
    off, exp, recv = ep.recv_segments(np.array([[1, 2], [0, 4]]))
    assert off.tolist() == [0, 1, 3, 3, 7]
    assert exp.tolist() == [0, 1, 0, 1]
    assert recv == [3, 4]
    with pytest.raises(ValueError):
        ep.expert_range(0, 3, 8)


def _rank_main(rank, world, port, case, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle as O
    from synthetic import MoEShape, make_inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T_loc, d, E, K, dff, S = case
        full = MoEShape("ep", T_loc * world, d, E, K, dff, n_shared=S, d_ff_shared=64 if S else 0, dtype=1,
                        zipf_logit_bias=True)
        inp = {k: (None if v is None else O.to_f64(v)) for k, v in make_inputs(full, seed=5, device="cpu").items()}
        mine = slice(rank * T_loc, (rank + 1) * T_loc)
        loc = full.replace(T=T_loc)
        inp_loc = dict(inp, x=inp["x"][mine])
        rt = O.route(loc, inp_loc)
        plan = rt["plan"]
        # dispatched rows, grouped by expert (hence by owner)
        x_disp = inp_loc["x"][plan["row_slot"] // K]
        counts = torch.as_tensor(plan["counts"].astype(np.int32))
        e_loc = E // world
        recv_counts = ep.exchange(counts, [e_loc] * world, [e_loc] * world)
        send = ep.send_splits(plan["counts"], world)
        seg_off, seg_exp, recv = ep.recv_segments(recv_counts.numpy().reshape(world, e_loc))
        x_recv = ep.exchange(torch.as_tensor(x_disp), send, recv).numpy()
        lo, hi = ep.expert_range(rank, world, E)
        y_recv = np.zeros_like(x_recv)
        for i in range(len(seg_exp)):
            a, b = int(seg_off[i]), int(seg_off[i + 1])
            if b > a:
                W1, b1, W2, b2 = O.expert_weights(inp, "W", lo + int(seg_exp[i]), False)
                y_recv[a:b] = O.expert_ffn(x_recv[a:b], W1, b1, W2, b2)
        y = ep.exchange(torch.as_tensor(y_recv), recv, send).numpy()
        # combine: gates * the slot's returned row, plus the shared experts
        out = np.zeros_like(inp_loc["x"])
        for t in range(T_loc):
            for k in range(K):
                r = plan["slot_row"][t, k]
                if r >= 0:
                    out[t] += rt["gates"][t, k] * y[r]
        for si in range(S):
            W1, b1, W2, b2 = O.expert_weights(inp, "Ws", si, False)
            out += O.expert_ffn(inp_loc["x"], W1, b1, W2, b2)
        want = O.layer_forward(loc, inp_loc)["out"]
        # balance statistics over all ranks' tokens
        c_all = torch.as_tensor(plan["counts"].astype(np.float64))
        dist.all_reduce(c_all)
        rt_all = O.route(full, inp)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"err": float(np.abs(out - want).max() / np.abs(want).max()),
                       "recv_rows": int(sum(recv)), "sent": send,
                       "f_ok": bool(np.allclose(c_all.numpy() / (full.T * K), rt_all["f"], rtol=0, atol=1e-15))}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [(2, (24, 64, 8, 2, 128, 1)), (4, (10, 64, 8, 3, 64, 0))])
def test_ep_exchange_matches_the_single_process_layer(tmp_path, world, case):
    mp.start_processes(_rank_main, args=(world, _free_port(), case, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    T_loc, _, _, K, _, _ = case
    for r in res:
        assert r["err"] < 1e-12, r
        assert r["f_ok"]
    # every slot went out once and came back once
    assert sum(sum(r["sent"]) for r in res) == sum(r["recv_rows"] for r in res) == world * T_loc * K

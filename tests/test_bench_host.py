"""Host logic of bench.py, on CPU: the cross-rank reduction of the replica
path on two gloo ranks, the whole-job throughput, the workload overrides,
the roofline arithmetic and the traffic table lookup."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synthetic import WORKLOADS  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_dir):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(times[rank], world)
        v = bench.job_throughput(4096, world, 10, t)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"t": t, "v": v}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_replica_timing_is_max_over_ranks_gloo(tmp_path, world):
    times = [3.25, 5.5]
    mp.start_processes(_rank_main, args=(world, _free_port(), times, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["t"] == max(times)                       # every rank sees the slowest replica
        assert r["v"] == pytest.approx(4096 * world * 10 / (max(times) * 1e-3))


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(2.0, 1) == 2.0
    assert bench.job_throughput(128, 1, 4, 2.0) == pytest.approx(128 * 4 / 2e-3)


def test_reference_arm_other_ranks_exit_without_output():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_set_overrides_build_a_reduced_case():
    args = bench.argparse.Namespace(config=4, set=["n_routed=64", "T=1024"])
    sh = bench.workload(args)
    assert (sh.n_routed, sh.T, sh.d_model, sh.top_k) == (64, 1024, 7168, 8)
    assert sh.name.endswith("[n_routed=64,T=1024]")
    assert bench.workload(bench.argparse.Namespace(config=2, set=[])) == WORKLOADS[2]


def test_roofline_work_per_step_closed_forms():
    import numpy as np
    sh = WORKLOADS[2]
    kept = np.full(sh.n_routed, sh.T * sh.top_k // sh.n_routed)
    R = int(kept.sum())
    assert bench.algorithmic_ffn(sh, R) == 4.0 * sh.d_model * sh.d_ff * R
    b, touched = bench.ffn_bytes(sh, kept)
    d, f = sh.d_model, sh.d_ff
    weights = sh.n_routed * (2 * d * f * 2 + 4 * (f + d))
    act = R * d * 2 + 2 * R * f * 2 + R * d * 2
    assert touched == sh.n_routed and b == weights + act
    # FP8: one byte per weight plus the fp32 block scales
    sh4 = WORKLOADS[4]
    kept4 = np.zeros(sh4.n_routed, dtype=np.int64)
    kept4[:3] = 10
    b4, t4 = bench.ffn_bytes(sh4, kept4)
    d, f, S, T = sh4.d_model, sh4.d_ff, sh4.n_shared, sh4.T
    w4 = 3 * (2 * d * f + 4 * (f + d)) + S * (2 * d * sh4.d_ff_shared + 4 * (sh4.d_ff_shared + d))
    w4 += 3 * 2 * (d // 128) * (f // 128) * 4 + S * 2 * (d // 128) * (sh4.d_ff_shared // 128) * 4
    R4 = 30
    act4 = (R4 + S * T) * d + 2 * (R4 * f + S * T * sh4.d_ff_shared) + (R4 + S * T) * d * 2
    assert t4 == 3 and b4 == w4 + act4


def test_traffic_lookup_requires_the_captured_sources():
    p = os.path.join(ROOT, "profiles", "grouped_ffn_traffic.json")
    entries = json.load(open(p))["entries"]
    assert entries
    for e in entries:
        assert bench.traffic_from_profile(e["workload"], e["kernel"], e["src_sha1"]) == e["dram_bytes_per_step"]
        assert bench.traffic_from_profile(e["workload"], e["kernel"], "0" * 40) is None
        assert bench.traffic_from_profile(e["workload"] + " other", e["kernel"], e["src_sha1"]) is None


def test_ffn_kernel_follows_dtype_and_pair_switch(monkeypatch):
    monkeypatch.delenv("MOE_GEMM_PAIR", raising=False)
    assert bench.ffn_kernel(WORKLOADS[1])[0] == "ffn_f32_kernel"
    assert bench.ffn_kernel(WORKLOADS[2])[0] == "grouped_ffn_bf16_pair_kernel"
    assert bench.ffn_kernel(WORKLOADS[4])[0] == "grouped_ffn_fp8_kernel"
    monkeypatch.setenv("MOE_GEMM_PAIR", "0")
    assert bench.ffn_kernel(WORKLOADS[2])[0] == "grouped_ffn_bf16_kernel"
    for cid in (1, 2, 4):
        for f in bench.ffn_kernel(WORKLOADS[cid])[1]:
            assert os.path.exists(os.path.join(bench.CSRC, f))


def test_stage_bytes_closed_forms():
    import numpy as np
    sh = WORKLOADS[2]
    T, d, E, K = sh.T, sh.d_model, sh.n_routed, sh.top_k
    kept = np.full(E, T * K // E)
    R = T * K
    b = bench.stage_bytes(sh, kept)
    assert b["route"] == T * d * 2 + E * d * 4 + T * K * 8 + (T // 32) * E * 4
    assert b["dispatch"] == T * K * 4 + T * d * 2 + R * d * 2 + T * K * 4 + R * 4 + (2 * E + 1) * 4
    assert b["combine"] == R * d * 2 + T * K * 8 + T * d * 2


def test_headline_is_the_v3_prefill_with_the_others_nested():
    import bench
    ns = bench.argparse.Namespace
    # the default headline is the largest single-GPU workload: V3 prefill, FP8
    import sys
    old = sys.argv
    try:
        sys.argv = ["bench.py"]
        args = bench.parse()
    finally:
        sys.argv = old
    assert args.config == 4 and args.workloads == "all"
    assert "v3-prefill" in bench.workload(args).name
    assert bench.other_workloads(args) == [1, 2, 3, 5]
    assert bench.other_workloads(ns(config=2, workloads="none", set=[])) == []
    assert bench.other_workloads(ns(config=4, workloads="2,3,4", set=[])) == [2, 3]
    # a reduced profiling case (--set) never carries nested workloads
    assert bench.other_workloads(ns(config=4, workloads="all", set=["T=1024"])) == []


def test_weight_bytes_of_the_workloads():
    import bench
    from synthetic import WORKLOADS
    # 2 x 7168 x (256 + 1) x 2048 e4m3 bytes
    assert bench.weight_bytes(WORKLOADS[4]) == 2 * 7168 * 257 * 2048
    # Mixtral shape: 2 x 4096 x 8 x 14336 bf16 values
    assert bench.weight_bytes(WORKLOADS[2]) == 2 * 4096 * 8 * 14336 * 2
    assert bench.weight_bytes(WORKLOADS[1]) < 126e6 < bench.weight_bytes(WORKLOADS[3])

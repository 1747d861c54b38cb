#!/usr/bin/env python
"""Benchmark of the sparse MoE FFN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4] [--workloads all|none|2,3]
                    [--impl ours|reference]

A step is one pass of the whole layer (router, dispatch, expert FFN grouped
GEMMs, combine, balance statistics) over one batch of seeded synthetic input
that is already resident in HBM.  The headline workload is the largest one
that fits one GPU: the DeepSeek-V3-shaped prefill layer (T=4096, d=7168, 256
experts, top-8, d_ff=2048, one shared expert, FP8 e4m3 dispatch and weights
with block scales, bf16 combine).  The other four workloads (tiny fp32,
Mixtral-8x7B-shaped bf16, DeepSeekMoE-style bf16 with a capacity limit, V3
decode with skewed routing) are measured the same way in the same run and
nested under "workloads".  Each timed step is bracketed by CUDA events on the
launching stream, with a 256 MiB write between steps (outside the events) to
flush L2.  Under torchrun each rank runs an independent replica (the layer
forward has no cross-GPU exchange); the time is the max over ranks and the
value counts the tokens of all ranks.

One JSON line on rank 0: tokens/s plus the grouped-GEMM roofline, the
per-stage HBM fractions, the CPU oracle baseline (rank 0, N=1), an end-to-end
figure through the public API with host buffers, and the SM clocks sampled
during the timed region; the same fields per nested workload.  For the fp32
and bf16 workloads the run also times the layer backward on the same batch
("backward": tokens/s, and for bf16 its expert GEMMs' TFLOP/s against the
tensor peak).

--impl reference times the CPU oracle (the reference implementation of this
repository: a plain fp64 restatement of the pages) on bounded token samples
of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s; grouped-GEMM TFLOP/s and HBM GB/s as % of B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Oracle tokens per CPU-baseline sample (about 10-30 s of host work; the whole
# batch where that fits) and per step of the reference arm (a fraction of a
# second to a few seconds, so that a default --steps/--warmup run of the
# reference arm ends within a few minutes).
CPU_SAMPLE = {1: 64, 2: 4096, 3: 8192, 4: 16, 5: 64}
REF_SAMPLE = {1: 64, 2: 32, 3: 64, 4: 1, 5: 4}
L2_FLUSH_BYTES = 256 << 20
STAGES = ["route", "dispatch", "expert_ffn", "combine", "balance"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=4, help="headline workload (1-5)")
    ap.add_argument("--workloads", default="all",
                    help="other workloads measured in the same run and nested in the line: "
                         "'all' (the four others), 'none', or a comma list such as '2,3'")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE",
                    help="override a field of the workload shape (e.g. n_routed=64); for profiling "
                         "reduced cases, never for the reported workload")
    return ap.parse_args()


def workload(args):
    from synthetic import WORKLOADS
    sh = WORKLOADS[args.config]
    if args.set:
        kw = {}
        for item in args.set:
            k, v = item.split("=", 1)
            cur = getattr(sh, k)
            kw[k] = type(cur)(float(v)) if isinstance(cur, (int, float)) and not isinstance(cur, bool) else type(cur)(v)
        sh = sh.replace(**kw)
        sh = sh.replace(name=sh.name + " [" + ",".join(args.set) + "]")
    return sh


def other_workloads(args):
    """The workloads measured after the headline one, in ascending order."""
    if args.set or args.workloads == "none":
        return []
    if args.workloads == "all":
        ids = [1, 2, 3, 4, 5]
    else:
        ids = sorted({int(v) for v in args.workloads.split(",") if v.strip()})
    return [c for c in ids if c != args.config]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def probe_fp8_peak(dev, n=8192, iters=10):
    """Dense FP8 tensor throughput of this GPU, measured once with a library
    GEMM (torch._scaled_mm, e4m3 x e4m3 -> bf16, n^3): a denominator probe for
    the FP8 expert GEMMs' tensor fraction, never on the measured path.
    Returns TFLOP/s, or None where the library call is unavailable."""
    import torch
    try:
        g = torch.Generator(device=dev).manual_seed(1)
        a = torch.randn((n, n), device=dev, generator=g).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), device=dev, generator=g).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev, dtype=torch.float32)
        for _ in range(3):
            torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record()
        for _ in range(iters):
            torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / iters
        del a, b
        return round(2.0 * n ** 3 / (ms * 1e-3) / 1e12, 1)
    except Exception:   # a probe: its absence leaves the field null
        return None


def max_over_ranks(ms, world, device=None):
    """The largest of the ranks' times (every rank returns it); the job is as
    slow as its slowest replica.  Works on the nccl (CUDA tensor) and gloo
    (CPU tensor) backends."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step, world, steps, total_ms):
    """Whole-job tokens/s: the tokens of all ranks over all timed steps,
    divided by the (max-over-ranks) time of those steps."""
    return tokens_per_rank_step * world * steps / (total_ms * 1e-3)


def workload_config(sh, seed, parallelism):
    return {"workload": sh.name, "T": sh.T, "d_model": sh.d_model, "n_routed": sh.n_routed,
            "top_k": sh.top_k, "d_ff": sh.d_ff, "n_shared": sh.n_shared, "d_ff_shared": sh.d_ff_shared,
            "capacity_factor": sh.capacity_factor, "seed": seed, "parallelism": parallelism,
            "l2": ("n/a (host oracle)" if parallelism == "cpu"
                   else "value: flushed between timed steps (256 MiB write, outside the timed events); "
                        "e2e: not flushed, the expert weights read every step "
                        f"({weight_bytes(sh) / 1e9:.2f} GB) exceed the 126 MB L2" +
                        (" (this tiny workload fits in L2)" if weight_bytes(sh) < 126e6 else ""))}


def weight_bytes(sh):
    """Bytes of all routed and shared expert weights of the layer."""
    wb = {0: 4, 1: 2, 2: 1}[sh.dtype]
    return 2 * sh.d_model * (sh.n_routed * sh.d_ff + sh.n_shared * sh.d_ff_shared) * wb


def dtype_name(sh):
    return {0: "f32", 1: "bf16", 2: "fp8-e4m3 (bf16 combine)"}[sh.dtype]


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"moe_clocks_{os.getpid()}.csv")
        self.marks = []

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=timestamp," + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except Exception:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        t0, t1 = (self.marks[0], self.marks[-1]) if len(self.marks) >= 2 else (0, 1e18)
        sel = [r for r in rows if t0 - 1 <= r[0] <= t1 + 1] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in sel for i in range(4) if r[3][i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in sel), "sm_max_mhz": max(r[2] for r in sel),
                "reasons": reasons, "samples": len(sel)}


# ----------------------------------------------------------------------------- oracle timing

def oracle_inputs_on_host(inp):
    """The inputs as the oracle reads them: on the host, fp32/bf16 values
    widened to fp64 numpy once (exact) so that the timed oracle calls do not
    re-convert the weights each step; FP8 codes stay as stored (their decode
    and block scaling are part of what the oracle computes)."""
    import torch
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif v.dtype in (torch.float32, torch.bfloat16, torch.float16):
            out[k] = v.detach().to("cpu", torch.float64).numpy()
        else:
            out[k] = v.detach().cpu()
    return out


def time_oracle(sh, host_inp, n_tokens, seed):
    import numpy as np
    import oracle as O
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(sh.T, size=min(n_tokens, sh.T), replace=False))
    t0 = time.perf_counter()
    O.layer_forward(sh, host_inp, tokens=toks)
    dt = time.perf_counter() - t0
    return len(toks), dt


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- our arm

def algorithmic_ffn(sh, kept_sum):
    """FLOPs and bytes of the expert FFN stage (both grouped GEMMs) for one
    step: real rows only.  Bytes: weights and biases of every expert that has
    rows, the dispatched activations read, the hidden activations written and
    read, the expert outputs written."""
    d, dff, S, T = sh.d_model, sh.d_ff, sh.n_shared, sh.T
    flops = 4.0 * d * dff * kept_sum + 4.0 * d * sh.d_ff_shared * S * T
    return flops


def ffn_bytes(sh, kept):
    d, dff, S, T, dfs = sh.d_model, sh.d_ff, sh.n_shared, sh.T, sh.d_ff_shared
    wb = {0: 4, 1: 2, 2: 1}[sh.dtype]
    ab = {0: 4, 1: 2, 2: 1}[sh.dtype]
    ob = 4 if sh.dtype == 0 else 2
    touched = int((kept > 0).sum())
    R = int(kept.sum())
    w = touched * (2 * d * dff * wb + 4 * (dff + d)) + S * (2 * d * dfs * wb + 4 * (dfs + d))
    if sh.dtype == 2:
        w += touched * 2 * (d // 128) * (dff // 128) * 4 + S * 2 * (d // 128) * (dfs // 128) * 4
    act = (R + S * T) * d * ab + 2 * (R * dff + S * T * dfs) * ab + (R + S * T) * d * ob
    return float(w + act), touched


def stage_bytes(sh, kept):
    """Algorithmic HBM bytes per step of the memory-bound stages: every
    operand read once and every result written once.
      route:    x, W_r (fp32), the logit bias, topk_idx + gates, the partial
                sums of s per 32-token block
      dispatch: topk_idx, x once, the dispatched rows (+ FP8 scales, + the
                quantised x of the shared experts), the slot maps
      combine:  the kept routed rows and the shared rows of y, gates and
                slot map, the layer output"""
    T, d, E, K, S = sh.T, sh.d_model, sh.n_routed, sh.top_k, sh.n_shared
    bx = {0: 4, 1: 2, 2: 2}[sh.dtype]          # x / y / out element bytes
    bq = {0: 4, 1: 2, 2: 1}[sh.dtype]          # dispatched row element bytes
    R = int(kept.sum())
    route = T * d * bx + E * d * 4 + (E * 4 if sh.zipf_logit_bias else 0) + T * K * 8 + ((T + 31) // 32) * E * 4
    disp = T * K * 4 + T * d * bx + R * d * bq + T * K * 4 + R * 4 + (2 * E + 1) * 4
    if sh.dtype == 2:
        disp += R * (d // 128) * 4
        if S > 0:
            disp += T * d + T * (d // 128) * 4
    comb = R * d * bx + S * T * d * bx + T * K * 8 + T * d * bx
    return {"route": float(route), "dispatch": float(disp), "combine": float(comb)}


CSRC = os.path.join(ROOT, "sparse_mixture_experts_20_b200", "csrc")


def ffn_kernel(sh):
    """(kernel name, source files) of the grouped FFN kernel the library runs
    for this dtype (the bf16 CTA-pair kernel unless MOE_GEMM_PAIR=0)."""
    if sh.dtype == 0:
        return "ffn_f32_kernel", ["ffn_f32.cu"]
    if sh.dtype == 2:
        return "grouped_ffn_fp8_kernel", ["ffn_fp8.cu", "ffn_common.cuh", "common.cuh"]
    if os.environ.get("MOE_GEMM_PAIR", "1") == "0":
        return "grouped_ffn_bf16_kernel", ["ffn_tc.cu", "ffn_common.cuh", "common.cuh"]
    return "grouped_ffn_bf16_pair_kernel", ["ffn_tc2.cu", "ffn_common.cuh", "common.cuh"]


def src_hash(files):
    h = hashlib.sha1()
    for f in files:
        h.update(open(os.path.join(CSRC, f), "rb").read())
    return h.hexdigest()


def stage_traffic(workload_name, stage):
    """DRAM bytes (read + write) per step of a memory-bound stage's kernels,
    from the committed ncu summary profiles/stage_traffic.json; None unless
    it was captured on this workload with that stage's sources unchanged."""
    p = os.path.join(ROOT, "profiles", "stage_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        for e in json.load(open(p)).get("entries", []):
            if e.get("workload") == workload_name and e.get("stage") == stage and \
                    e.get("src_sha1") == src_hash(e.get("sources", [])):
                return e.get("dram_bytes_per_step")
    except Exception:
        return None
    return None


def traffic_from_profile(workload_name, kernel, sha):
    """DRAM bytes (read + write) of the grouped FFN launches of one step, from
    the committed ncu summary; None unless it was captured on this workload
    with the kernel sources unchanged since."""
    p = os.path.join(ROOT, "profiles", "grouped_ffn_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        for e in json.load(open(p)).get("entries", []):
            if e.get("workload") == workload_name and e.get("kernel") == kernel and e.get("src_sha1") == sha:
                return e.get("dram_bytes_per_step")
    except Exception:
        return None
    return None


def measure_workload(args, cid, sh, dev, world, rank, local, peaks, peak_src, cpu_baseline):
    """Times K steps of one workload on this rank (max over ranks) and returns
    its fields: tokens/s, per-stage times, the grouped-GEMM roofline, the
    stage HBM fractions, the end-to-end figure, routing statistics, clocks,
    and (rank 0 at N=1, if asked) the CPU oracle baseline."""
    import numpy as np
    import torch

    import sparse_mixture_experts_20_b200 as M
    from synthetic import make_inputs

    inp = make_inputs(sh, seed=args.seed + rank, device=dev)
    cfg = M.make_config(sh)
    T, K, E, d = sh.T, sh.top_k, sh.n_routed, sh.d_model
    cap, r_cap, x_rows, y_rows = M.moe_buffer_rows(cfg)
    fp8 = sh.dtype == 2
    act = torch.float32 if sh.dtype == 0 else torch.bfloat16
    ws = torch.empty(M.moe_workspace_size(cfg), dtype=torch.uint8, device=dev)
    M.moe_workspace_init(cfg, ws)
    i32 = dict(dtype=torch.int32, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    b = {
        "topk_idx": torch.empty((T, K), **i32), "gates": torch.empty((T, K), **f32),
        "counts": torch.empty(E, **i32), "kept": torch.empty(E, **i32), "offsets": torch.empty(E + 1, **i32),
        "slot_row": torch.empty((T, K), **i32), "row_slot": torch.empty(max(r_cap, 1), **i32),
        "x_disp": torch.empty((x_rows, d), dtype=torch.uint8 if fp8 else act, device=dev),
        "x_disp_scales": torch.empty((x_rows, d // 128), **f32) if fp8 else None,
        "y": torch.empty((y_rows, d), dtype=act, device=dev), "out": torch.empty((T, d), dtype=act, device=dev),
        "f": torch.empty(E, **f32), "P": torch.empty(E, **f32), "loss": torch.empty(1, **f32),
    }
    g = inp.get
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    n_stage = len(STAGES)

    def step(ev):
        ev[0].record(stream)
        M.moe_route(cfg, inp["x"], g("W_r"), g("logit_bias"), b["topk_idx"], b["gates"], None, ws)
        ev[1].record(stream)
        M.moe_dispatch(cfg, inp["x"], b["topk_idx"], b["counts"], b["kept"], b["offsets"], b["slot_row"],
                       b["row_slot"], b["x_disp"], b["x_disp_scales"], ws)
        ev[2].record(stream)
        M.moe_expert_ffn(cfg, inp["x"], b["x_disp"], b["x_disp_scales"], b["offsets"], g("W1"), g("W1_scales"),
                         g("b1"), g("W2"), g("W2_scales"), g("b2"), g("Ws1"), g("Ws1_scales"), g("bs1"),
                         g("Ws2"), g("Ws2_scales"), g("bs2"), b["y"], ws)
        ev[3].record(stream)
        M.moe_combine(cfg, b["y"], b["gates"], b["slot_row"], b["out"], x=inp["x"])
        ev[4].record(stream)
        M.moe_balance_stats(cfg, b["counts"], ws, b["f"], b["P"], b["loss"])
        ev[5].record(stream)

    layer = M.MoELayer(cfg, inp, device=dev)
    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(args.warmup):
        flush.zero_()
        step([torch.cuda.Event(enable_timing=True) for _ in range(n_stage + 1)])
        flush.zero_()
        layer.forward(inp["x"])
    torch.cuda.synchronize(dev)
    assert M.moe_get_device_status(cfg, ws) == 0, "device status after warm-up"
    assert layer.device_status() == 0, "device status after warm-up"

    # ---- the timed steps: one moe_layer_forward call each (the whole layer,
    # inputs resident in HBM), L2 flushed before each step outside the events
    lev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world, local)
    torch.cuda.synchronize(dev)
    sampler.mark()
    launches0 = M.moe_kernel_launches()
    for k in range(args.steps):
        flush.zero_()
        lev[k][0].record(stream)
        layer.forward(inp["x"])
        lev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    launches = M.moe_kernel_launches() - launches0
    barrier(world, local)
    layer_ms = np.array([a.elapsed_time(c) for a, c in lev])
    total_ms = max_over_ranks(float(layer_ms.sum()), world, dev)

    # ---- the same steps through the stage entry points with an event between
    # stages: the per-stage times, the grouped-GEMM roofline and the stage HBM
    # fractions
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_stage + 1)] for _ in range(args.steps)]
    barrier(world, local)
    torch.cuda.synchronize(dev)
    for k in range(args.steps):
        flush.zero_()
        step(evs[k])
    torch.cuda.synchronize(dev)
    sampler.mark()
    barrier(world, local)
    stage_ms = np.array([[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(n_stage)]
                         for k in range(args.steps)])
    staged_total_ms = max_over_ranks(float(stage_ms.sum()), world, dev)
    kept = b["kept"].cpu().numpy()
    counts = b["counts"].cpu().numpy()
    status = M.moe_get_device_status(cfg, ws) | layer.device_status()
    assert torch.equal(layer.topk_idx, b["topk_idx"]), "the layer call and the stage calls route alike"
    bwd = None
    if sh.dtype != 2:
        bwd = measure_backward(args, sh, cfg, inp, b, ws, dev, world, local, stream, flush, int(kept.sum()),
                               peaks, peak_src)
        sampler.mark()
    del b

    # ---- end to end through the public API: pinned host x in, out + loss back
    x_h = inp["x"].cpu().pin_memory()
    out_h = torch.empty((T, d), dtype=act).pin_memory()
    loss_h = torch.empty(1, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(inp["x"])
    for _ in range(max(1, min(args.warmup, 3))):
        x_dev.copy_(x_h, non_blocking=True)
        layer.forward(x_dev)
    # serial: copy in, compute, copy back, one after another on one stream
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world, local)
    torch.cuda.synchronize(dev)
    for k in range(args.steps):
        e2e_ev[k][0].record(stream)
        x_dev.copy_(x_h, non_blocking=True)
        out, f, P, loss = layer.forward(x_dev)
        out_h.copy_(out, non_blocking=True)
        loss_h.copy_(loss, non_blocking=True)
        e2e_ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, local)
    e2e_serial_ms = max_over_ranks(float(sum(a.elapsed_time(c) for a, c in e2e_ev)), world, dev)
    # pipelined: MoELayer.forward_host_batches overlaps batch k's compute with
    # batch k+1's host->device and batch k-1's device->host copies; every
    # batch's copies are inside the timed region (first copy in .. last copy out)
    layer.forward_host_batches([x_h] * 3, [out_h] * 3, [loss_h] * 3)
    barrier(world, local)
    torch.cuda.synchronize(dev)
    ev0, ev1 = layer.forward_host_batches([x_h] * args.steps, [out_h] * args.steps, [loss_h] * args.steps)
    torch.cuda.synchronize(dev)
    barrier(world, local)
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    clocks = sampler.stop()
    del layer, flush

    ffn_ms = float(stage_ms[:, STAGES.index("expert_ffn")].mean())
    flops = algorithmic_ffn(sh, int(kept.sum()))
    fbytes, touched = ffn_bytes(sh, kept)
    roof = ffn_roofline(sh, flops, fbytes, touched, ffn_ms, peaks, peak_src)

    sb = stage_bytes(sh, kept)
    stages_hbm = {}
    for i, name in enumerate(STAGES):
        if name in sb:
            ms_i = float(stage_ms[:, i].mean())
            gbs = sb[name] / (ms_i * 1e-3) / 1e9
            stages_hbm[name] = {"bytes": sb[name], "gbs": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4),
                                "traffic": stage_traffic(sh.name, name)}
    res = {
        "value": round(job_throughput(T, world, args.steps, total_ms), 1), "unit": "tokens/s",
        "ms_per_step": round(total_ms / args.steps, 4),
        "dtype": dtype_name(sh),
        "config": workload_config(sh, args.seed, "replicas" if world > 1 else "single"),
        "timing": "value and ms_per_step: moe_layer_forward per step (CUDA events around the call); "
                  "stages_ms: the same step through the five stage entry points with an event between stages "
                  f"({staged_total_ms / args.steps:.4f} ms per step that way)",
        "stages_ms": {n: round(float(stage_ms[:, i].mean()), 4) for i, n in enumerate(STAGES)},
        "grouped_gemm_tflops": round(flops / (ffn_ms * 1e-3) / 1e12, 1),
        "stages_hbm": stages_hbm,
        "roofline": roof,
        "e2e": {"value": round(job_throughput(T, world, args.steps, e2e_ms), 1), "unit": "tokens/s",
                "copies": "pinned host x in and out + loss back every step, on their own streams, "
                          "overlapping the neighbouring steps' compute (MoELayer.forward_host_batches)",
                "serial_value": round(job_throughput(T, world, args.steps, e2e_serial_ms), 1),
                "h2d_bytes_per_step": int(inp["x"].numel() * inp["x"].element_size()),
                "d2h_bytes_per_step": int(T * d * (4 if sh.dtype == 0 else 2) + 4)},
        "gpu_launches": launches,
        "routing": {"max_load": int(counts.max()), "mean_load": float(counts.mean()),
                    "experts_touched": int((counts > 0).sum()), "dropped": int(counts.sum() - kept.sum())},
        "device_status": status,
        "clocks": clocks,
    }
    if bwd is not None:
        res["backward"] = bwd
    if cpu_baseline and rank == 0 and world == 1:
        host = oracle_inputs_on_host(inp)
        # passes over the sample until about 10 s of host work (at least one)
        n_tot, dt_tot, passes = 0, 0.0, 0
        while passes == 0 or (dt_tot < 10.0 and passes < 16):
            n, dt = time_oracle(sh, host, CPU_SAMPLE.get(cid, 64), args.seed + passes)
            n_tot, dt_tot, passes = n_tot + n, dt_tot + dt, passes + 1
        res["cpu_baseline"] = {"value": round(n_tot / dt_tot, 3), "unit": "tokens/s", "cores": oracle_threads(),
                               "kind": "oracle",
                               "sample": f"{passes} pass(es) of {n} of {T} tokens (routing of all {T} each pass), "
                                         f"fp64 numpy, {dt_tot:.1f} s; fp32/bf16 inputs widened to fp64 once "
                                         "before timing"}
        del host
    del inp
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return res


def backward_flops(sh, kept_sum):
    """Tensor-core work of one layer backward: per routed row and per shared
    expert's token five d x d_ff products (recompute of z, dh, dx, dW2, dW1)
    of 2 flop per multiply-add."""
    return 10.0 * sh.d_model * (kept_sum * sh.d_ff + sh.n_shared * sh.T * sh.d_ff_shared)


def measure_backward(args, sh, cfg, inp, b, ws, dev, world, local, stream, flush, kept_sum, peaks, peak_src):
    """K timed calls of moe_layer_backward on the forward results of this
    batch (fp32 gradients of <dout, out> + L_balance), L2 flushed between
    calls outside the events; tokens/s and the expert GEMMs' flops over the
    whole call against the bf16 tensor peak."""
    import numpy as np
    import torch

    import sparse_mixture_experts_20_b200 as M
    T, d, E = sh.T, sh.d_model, sh.n_routed
    f32 = dict(dtype=torch.float32, device=dev)
    logits = torch.empty((T, E), **f32)
    M.moe_route(cfg, inp["x"], inp.get("W_r"), inp.get("logit_bias"), b["topk_idx"], b["gates"], logits, ws)
    gen = torch.Generator(device=dev).manual_seed(args.seed + 17)
    dout = torch.randn((T, d), generator=gen, device=dev, dtype=torch.float32).to(inp["x"].dtype)
    t = {k: inp.get(k) for k in ("x", "W_r", "W1", "b1", "W2", "b2", "Ws1", "bs1", "Ws2", "bs2")}
    t.update({k: b[k] for k in ("topk_idx", "gates", "counts", "offsets", "slot_row", "row_slot", "x_disp", "y")})
    t.update(logits=logits, dout=dout, dx=torch.empty((T, d), **f32), dW_r=torch.empty((E, d), **f32),
             dW1=torch.empty(inp["W1"].shape, **f32), db1=torch.empty(inp["b1"].shape, **f32),
             dW2=torch.empty(inp["W2"].shape, **f32), db2=torch.empty(inp["b2"].shape, **f32))
    if inp.get("logit_bias") is not None:
        t["d_logit_bias"] = torch.empty(E, **f32)
    if sh.n_shared:
        for k in ("Ws1", "bs1", "Ws2", "bs2"):
            t["d" + k] = torch.empty(inp[k].shape, **f32)
    bws = torch.empty(M.moe_backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    for _ in range(max(3, min(args.warmup, 5))):
        flush.zero_()
        M.moe_layer_backward(cfg, 1.0, t, bws)
    torch.cuda.synchronize(dev)
    assert bws[:4].view(torch.int32).item() == 0, "backward device status after warm-up"
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world, local)
    torch.cuda.synchronize(dev)
    l0 = M.moe_kernel_launches()
    for k in range(args.steps):
        flush.zero_()
        ev[k][0].record(stream)
        M.moe_layer_backward(cfg, 1.0, t, bws)
        ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    launches = M.moe_kernel_launches() - l0
    barrier(world, local)
    ms = np.array([a.elapsed_time(c) for a, c in ev])
    total = max_over_ranks(float(ms.sum()), world, dev)
    status = int(bws[:4].view(torch.int32).item())
    flops = backward_flops(sh, kept_sum)
    per = total / args.steps
    ach = flops / (per * 1e-3) / 1e12
    res = {"value": round(job_throughput(T, world, args.steps, total), 1), "unit": "tokens/s",
           "ms_per_step": round(per, 4),
           "what": "moe_layer_backward per step (gradients of x, W_r, bias, every expert's weights and biases, "
                   "fp32) on this batch's forward results; CUDA events around the call",
           "gpu_launches": launches, "device_status": status}
    if sh.dtype == 1:
        res["roofline"] = {"bound": "tensor", "achieved": round(ach, 1), "peak": peaks["bf16_tflops"],
                           "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops"], 4),
                           "peak_source": f"{peak_src} (bf16 burst)",
                           "frac_of_sustained_peak": round(ach / peaks["bf16_tflops_sustained"], 4)
                           if peaks.get("bf16_tflops_sustained") else None,
                           "kernel": "bwd_gemm_kernel (five launches: recompute, dz, dx, dW2, dW1); achieved = "
                                     "their algorithmic flops over the whole backward call",
                           "algorithmic": {"flops": flops}, "traffic": None}
    del t, bws, logits, dout
    return res


def barrier(world, local):
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])


def ffn_roofline(sh, flops, fbytes, touched, ffn_ms, peaks, peak_src):
    """Roofline of the grouped expert FFN (both launches of a step): the
    slower of the flops at the tensor peak and the bytes at the HBM peak
    binds; achieved is the algorithmic work over the CUDA-event time."""
    fp8 = sh.dtype == 2
    tens_peak = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
    t_tensor = flops / (tens_peak * 1e12)
    t_hbm = fbytes / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        ach = flops / (ffn_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": tens_peak, "unit": "TFLOP/s",
                "frac": round(ach / tens_peak, 4)}
    else:
        ach = fbytes / (ffn_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / peaks["hbm_gbs"], 4)}
    kname, kfiles = ffn_kernel(sh)
    roof["kernel"] = f"{kname} (both launches of a step: first and second layer)"
    roof["peak_source"] = (f"{peak_src} ({'bf16 burst x2 nominal fp8/bf16 ratio' if fp8 else 'bf16 burst'})"
                           if roof["bound"] == "tensor" else f"{peak_src} HBM copy")
    roof["traffic"] = traffic_from_profile(sh.name, kname, src_hash(kfiles))
    # the nominal B200 peaks the targets are written against (dense bf16
    # 2.25 PF, fp8 4.5 PF, HBM 8 TB/s), beside the measured ones
    spec = (4500.0 if fp8 else 2250.0) if roof["bound"] == "tensor" else 8000.0
    roof["frac_of_spec_peak"] = round(roof["achieved"] / spec, 4)
    if roof["bound"] == "tensor":
        # a dense GEMM at the 1 kW power cap runs below the burst clock: the
        # sustained measured peak, for context
        sus = peaks.get("bf16_tflops_sustained")
        if sus:
            sus = sus * (2.0 if fp8 else 1.0)
            roof["frac_of_sustained_peak"] = round(roof["achieved"] / sus, 4)
    if fp8:
        # the tensor side of the HBM-bound FP8 GEMMs, against a library FP8
        # GEMM's dense throughput measured on this GPU in the same run
        tfl = flops / (ffn_ms * 1e-3) / 1e12
        roof["tensor_tflops"] = round(tfl, 1)
        probe = peaks.get("fp8_tflops_probe")
        roof["tensor_frac_of_fp8_probe"] = round(tfl / probe, 4) if probe else None
    roof["algorithmic"] = {"flops": flops, "bytes": fbytes, "experts_touched": touched}
    return roof


def run_ours(args):
    import torch
    import torch.distributed as dist

    import sparse_mixture_experts_20_b200 as M
    from synthetic import WORKLOADS

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    M.lib()
    peaks, peak_src = load_peaks()
    peaks["fp8_tflops_probe"] = probe_fp8_peak(dev)
    head = measure_workload(args, args.config, workload(args), dev, world, rank, local, peaks, peak_src,
                            cpu_baseline=not args.no_cpu_baseline)
    nested = {}
    for cid in other_workloads(args):
        nested[str(cid)] = measure_workload(args, cid, WORKLOADS[cid], dev, world, rank, local, peaks, peak_src,
                                            cpu_baseline=False)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"],
                "data": "synthetic (seeded N(0,1) activations, N(0,1/fan_in) weights, N(0,0.01) biases)",
                "config": head["config"], "impl": "ours"}
        for k in ("timing", "stages_ms", "grouped_gemm_tflops", "stages_hbm", "roofline", "e2e", "gpu_launches",
                  "routing", "device_status", "clocks", "cpu_baseline", "backward"):
            if k in head:
                line[k] = head[k]
        line["peaks"] = {"source": peak_src, "hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
                         "fp8_tflops_probe": peaks["fp8_tflops_probe"],
                         "fp8_probe": "torch._scaled_mm e4m3 8192^3 -> bf16, 10 calls after 3, CUDA events"}
        if nested:
            line["workloads"] = nested
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch
    from synthetic import make_inputs
    sh = workload(args)
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    host = oracle_inputs_on_host(make_inputs(sh, seed=args.seed, device=gen_dev))
    n_tok = REF_SAMPLE.get(args.config, 16)
    for w in range(args.warmup):
        time_oracle(sh, host, n_tok, args.seed + 1000 + w)
    total_t, total_n = 0.0, 0
    for k in range(args.steps):
        n, dt = time_oracle(sh, host, n_tok, args.seed + k)
        total_t += dt
        total_n += n
    value = total_n / total_t
    cores = oracle_threads()
    sample = (f"{n_tok} of {sh.T} tokens per step (routing of all {sh.T}), fp64 numpy, "
              "fp32/bf16 inputs widened to fp64 once before timing")
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000 * total_t / args.steps, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": workload_config(sh, args.seed, "cpu"),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

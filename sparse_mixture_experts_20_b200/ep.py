"""Expert parallelism of the MoE layer over the ranks of a torch.distributed
process group (NCCL between GPUs; gloo works for the host-side plan).

"エキスパート並列（Expert Parallelism）" §推論フロー: the routed experts of a
layer are spread over GPUs; every token's rows travel to the GPU holding the
expert chosen for them and their outputs travel back.  "DeepSeek DeepEP"
§DeepEP とは: the dispatch carries FP8 rows (e4m3 codes with their 1x128
scales) and the combine bf16 rows.

Rank r of W ranks holds routed experts r*E_loc .. (r+1)*E_loc - 1 (E_loc =
n_routed / W), the router and the shared experts (replicated), and its own
batch of T tokens.  One forward:
  1. moe_route and moe_dispatch on the local batch over all n_routed experts:
     the dispatched rows (FP8 codes and scales, or bf16 / fp32 rows) come out
     grouped by expert, hence by the rank that owns the expert;
  2. every rank sends each owner the per-expert counts of the rows it will
     receive (all_to_all), then the rows themselves (one all_to_all per
     tensor, split by owner);
  3. moe_expert_ffn_segments runs the held experts on the received rows where
     they landed: one segment per (source rank, expert), in arrival order;
  4. the outputs travel back (all_to_all, bf16 / fp32) into the dispatched-row
     layout; moe_expert_ffn adds the shared experts' rows (no routed rows) and
     moe_combine sums gates * rows + shared rows per token;
  5. balance statistics over all ranks' tokens: f from the summed counts, P
     from the summed per-rank sums of s (all_reduce).
The split sizes of an all_to_all live on the host, so the counts are copied
there (one synchronisation per forward).  No capacity limit in this form (a
capacity would rank a slot among every rank's tokens at the expert's owner).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np


def expert_range(rank: int, world: int, n_routed: int) -> Tuple[int, int]:
    """[first, last + 1) of the routed experts rank `rank` holds."""
    if n_routed % world:
        raise ValueError(f"n_routed={n_routed} is not a multiple of the {world} ranks")
    e_loc = n_routed // world
    return rank * e_loc, (rank + 1) * e_loc


def send_splits(counts: Sequence[int], world: int) -> List[int]:
    """Rows this rank sends to each rank: its dispatched rows are grouped by
    expert, so the rows for rank r are those of r's experts, in order."""
    c = np.asarray(counts, np.int64)
    e_loc = len(c) // world
    return [int(c[r * e_loc:(r + 1) * e_loc].sum()) for r in range(world)]


def recv_segments(recv_counts: np.ndarray):
    """recv_counts (W, E_loc): rows source rank s sends for each held expert.
    Returns (seg_offsets (W*E_loc + 1), seg_expert (W*E_loc), recv_splits
    (W)): the received rows are source-major and, within a source, grouped by
    expert (its dispatch order), so segment s*E_loc + e holds source s's rows
    for held expert e."""
    rc = np.asarray(recv_counts, np.int64)
    world, e_loc = rc.shape
    flat = rc.reshape(-1)
    offsets = np.zeros(flat.size + 1, np.int64)
    np.cumsum(flat, out=offsets[1:])
    expert = np.tile(np.arange(e_loc, dtype=np.int64), world)
    return offsets, expert, [int(v) for v in rc.sum(axis=1)]


def exchange(t, send: Sequence[int], recv: Sequence[int], group=None, out=None):
    """all_to_all of the rows of t (rows along dim 0): send[r] rows to rank r,
    recv[r] rows from rank r, concatenated in rank order."""
    import torch
    import torch.distributed as dist
    if out is None:
        out = torch.empty((int(sum(recv)),) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_to_all_single(out, t.contiguous(), output_split_sizes=list(recv), input_split_sizes=list(send),
                           group=group)
    return out


class ExpertParallelMoE:
    """The MoE layer with its routed experts spread over the ranks of `group`.

    cfg: the layer (moe_config) with T = this rank's tokens per batch and
    n_routed = all routed experts (a multiple of the group size); no capacity.
    weights: W_r, logit_bias, the shared experts (as MoELayer) and W1, W1_scales,
    b1, W2, W2_scales, b2 of the held experts only (leading dimension E_loc).
    forward(x) returns (out, f, P, loss) like MoELayer.forward, f, P and loss
    over every rank's tokens."""

    def __init__(self, cfg, weights: dict, group=None, device="cuda"):
        import torch
        import torch.distributed as dist
        from . import (MOE_FP8_E4M3_BLOCK, MOE_F32, make_config, moe_buffer_rows, moe_workspace_init,
                       moe_workspace_size)
        if cfg.capacity_factor != 0.0:
            raise ValueError("expert parallelism in this form has no capacity limit")
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.lo, self.hi = expert_range(self.rank, self.world, cfg.n_routed)
        self.e_loc = self.hi - self.lo
        self.cfg = cfg
        self.w = weights
        self.dev = torch.device(device)
        dev = self.dev
        self.fp8 = cfg.dtype == MOE_FP8_E4M3_BLOCK
        act = torch.float32 if cfg.dtype == MOE_F32 else torch.bfloat16
        self.act = act
        T, K, E, d = cfg.T, cfg.top_k, cfg.n_routed, cfg.d_model
        cap, r_cap, x_rows, y_rows = moe_buffer_rows(cfg)
        self.r_cap = r_cap
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.ws = torch.empty(moe_workspace_size(cfg), dtype=torch.uint8, device=dev)
        moe_workspace_init(cfg, self.ws)
        self.topk_idx = torch.empty((T, K), **i32)
        self.gates = torch.empty((T, K), **f32)
        self.counts = torch.empty(E, **i32)
        self.kept = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.zero_offsets = torch.zeros(E + 1, **i32)
        self.slot_row = torch.empty((T, K), **i32)
        self.row_slot = torch.empty(max(r_cap, 1), **i32)
        self.x_disp = torch.empty((x_rows, d), dtype=torch.uint8 if self.fp8 else act, device=dev)
        self.x_disp_scales = torch.empty((x_rows, d // 128), **f32) if self.fp8 else None
        self.y = torch.empty((y_rows, d), dtype=act, device=dev)
        self.out = torch.empty((T, d), dtype=act, device=dev)
        self.f = torch.empty(E, **f32)
        self.P = torch.empty(E, **f32)
        self.loss = torch.empty(1, **f32)
        # the held experts see at most every rank's T*K rows
        self.recv_cap = self.world * T * K
        self.cfg_seg = make_config(T=self.recv_cap, d_model=d, n_routed=self.e_loc, top_k=1, d_ff=cfg.d_ff,
                                   dtype=cfg.dtype, alpha=cfg.alpha)
        self.ws_seg = torch.empty(moe_workspace_size(self.cfg_seg), dtype=torch.uint8, device=dev)
        moe_workspace_init(self.cfg_seg, self.ws_seg)
        self.x_recv = torch.empty((self.recv_cap, d), dtype=self.x_disp.dtype, device=dev)
        self.x_recv_scales = torch.empty((self.recv_cap, d // 128), **f32) if self.fp8 else None
        self.y_recv = torch.empty((self.recv_cap, d), dtype=act, device=dev)

    def forward(self, x):
        import torch
        import torch.distributed as dist
        from . import (moe_balance_stats, moe_combine, moe_dispatch, moe_expert_ffn, moe_expert_ffn_segments,
                       moe_route)
        cfg, w, g = self.cfg, self.w, self.w.get
        world = self.world
        moe_route(cfg, x, g("W_r"), g("logit_bias"), self.topk_idx, self.gates, None, self.ws)
        moe_dispatch(cfg, x, self.topk_idx, self.counts, self.kept, self.offsets, self.slot_row, self.row_slot,
                     self.x_disp, self.x_disp_scales, self.ws)
        # counts to the owners; split sizes on the host
        recv_counts = exchange(self.counts, [self.e_loc] * world, [self.e_loc] * world, self.group)
        counts_h = self.counts.cpu().numpy()
        rc_h = recv_counts.cpu().numpy().reshape(world, self.e_loc)
        send = send_splits(counts_h, world)
        seg_off, seg_exp, recv = recv_segments(rc_h)
        R = int(sum(send))
        n_recv = int(sum(recv))
        seg_off_d = torch.as_tensor(seg_off.astype(np.int32), device=self.dev)
        seg_exp_d = torch.as_tensor(seg_exp.astype(np.int32), device=self.dev)
        # rows to the owners (FP8: codes and scales)
        exchange(self.x_disp[:R], send, recv, self.group, out=self.x_recv[:n_recv])
        if self.fp8:
            exchange(self.x_disp_scales[:R], send, recv, self.group, out=self.x_recv_scales[:n_recv])
        if n_recv > 0:
            moe_expert_ffn_segments(self.cfg_seg, self.x_recv, self.x_recv_scales, seg_off_d, seg_exp_d,
                                    len(seg_exp), g("W1"), g("W1_scales"), g("b1"), g("W2"), g("W2_scales"),
                                    g("b2"), self.y_recv, self.ws_seg)
        # outputs back into the dispatched-row layout
        exchange(self.y_recv[:n_recv], recv, send, self.group, out=self.y[:R])
        if cfg.n_shared > 0:
            # no routed rows here (zero offsets): the shared experts only
            moe_expert_ffn(cfg, x, self.x_disp, self.x_disp_scales, self.zero_offsets, g("W1"), g("W1_scales"),
                           g("b1"), g("W2"), g("W2_scales"), g("b2"), g("Ws1"), g("Ws1_scales"), g("bs1"),
                           g("Ws2"), g("Ws2_scales"), g("bs2"), self.y, self.ws)
        moe_combine(cfg, self.y, self.gates, self.slot_row, self.out, x=x)
        # balance statistics over all ranks: f_j = sum counts / (T_all K),
        # P_j = sum over ranks of T * P_local / T_all
        moe_balance_stats(cfg, self.counts, self.ws, self.f, self.P, self.loss)
        T_all = float(cfg.T * world)
        counts_all = self.counts.to(torch.float64)
        p_sum = self.P.to(torch.float64) * cfg.T
        dist.all_reduce(counts_all, group=self.group)
        dist.all_reduce(p_sum, group=self.group)
        f = counts_all / (T_all * cfg.top_k)
        P = p_sum / T_all
        self.f.copy_(f)
        self.P.copy_(P)
        self.loss.copy_((cfg.alpha * cfg.n_routed * (f * P).sum()).reshape(1))
        return self.out, self.f, self.P, self.loss

    def device_status(self) -> int:
        from . import moe_get_device_status
        return moe_get_device_status(self.cfg, self.ws) | moe_get_device_status(self.cfg_seg, self.ws_seg)

"""Sparse MoE FFN layer forward on one B200: Python binding of libmoe_b200.so.

The binding only marshals arguments (torch tensors -> device pointers, the
current CUDA stream) into the C ABI declared in include/moe_b200.h; every step
of the layer runs in the library's CUDA kernels.  There is no CPU or PyTorch
fallback: if the shared library is missing, importing the entry points raises.

Entry points (same names as the C ABI): moe_workspace_size, moe_buffer_rows,
moe_workspace_init, moe_get_device_status, moe_route, moe_dispatch,
moe_expert_ffn, moe_combine, moe_balance_stats, moe_layer_forward,
moe_selftest_wait_timeout.  `MoELayer` bundles a config, its workspace and
its weights for the common whole-layer call.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_BAD_ROUTING = 4
MOE_ERR_DEVICE_TIMEOUT = 5
MOE_DEV_BAD_ROUTING = 0x1
MOE_DEV_TIMEOUT = 0x2
MOE_F32, MOE_BF16, MOE_FP8_E4M3_BLOCK = 0, 1, 2
MOE_BIAS_LOGITS, MOE_BIAS_SELECTION = 0, 1
MOE_PRIORITY_TOKEN, MOE_PRIORITY_SLOT = 0, 1
MOE_OVERFLOW_DROP, MOE_OVERFLOW_PASS = 0, 1

EXPORTED = (
    "moe_workspace_size", "moe_buffer_rows", "moe_workspace_init", "moe_get_device_status",
    "moe_last_cuda_error", "moe_status_string", "moe_route", "moe_dispatch", "moe_expert_ffn",
    "moe_combine", "moe_balance_stats", "moe_layer_forward", "moe_selftest_wait_timeout",
    "moe_dispatch_noalloc", "moe_kernel_launches", "moe_backward_workspace_size", "moe_layer_backward",
    "moe_expert_ffn_segments",
)


class moe_config(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_routed", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("n_shared", ctypes.c_int32),
        ("d_ff_shared", ctypes.c_int32), ("capacity_factor", ctypes.c_float),
        ("alpha", ctypes.c_float), ("dtype", ctypes.c_int32), ("bias_mode", ctypes.c_int32),
        ("capacity_priority", ctypes.c_int32), ("overflow_mode", ctypes.c_int32),
    ]


class moe_backward_io(ctypes.Structure):
    """Pointers of moe_layer_backward, in the header's order."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "x", "W_r", "W1", "b1", "W2", "b2", "Ws1", "bs1", "Ws2", "bs2",
        "logits", "topk_idx", "gates", "counts", "offsets", "slot_row", "row_slot", "x_disp", "y",
        "dout",
        "dx", "dW_r", "d_logit_bias", "dW1", "db1", "dW2", "db2", "dWs1", "dbs1", "dWs2", "dbs2")]


BACKWARD_IO_FIELDS = tuple(n for n, _ in moe_backward_io._fields_)


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = lib().moe_status_string(status).decode()
        extra = ""
        if status == MOE_ERR_CUDA:
            extra = f" (cudaError {lib().moe_last_cuda_error()})"
        super().__init__(f"{where}: {name}{extra}")


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded shared library.  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m sparse_mixture_experts_20_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        cfgp = ctypes.POINTER(moe_config)
        I = ctypes.c_int
        sig = {
            "moe_workspace_size": [cfgp, ctypes.POINTER(ctypes.c_size_t)],
            "moe_buffer_rows": [cfgp] + [ctypes.POINTER(ctypes.c_int32)] * 4,
            "moe_workspace_init": [cfgp, P, P],
            "moe_get_device_status": [cfgp, P, P, ctypes.POINTER(ctypes.c_int32), ctypes.c_int32],
            "moe_last_cuda_error": [],
            "moe_status_string": [I],
            "moe_route": [cfgp, P, P, P, P, P, P, P, P],
            "moe_dispatch": [cfgp, P, P, P, P, P, P, P, P, P, P, P],
            "moe_expert_ffn": [cfgp] + [P] * 19,
            "moe_combine": [cfgp, P, P, P, P, P, P],
            "moe_balance_stats": [cfgp, P, P, P, P, P, P],
            "moe_layer_forward": [cfgp] + [P] * 24,
            "moe_selftest_wait_timeout": [cfgp, ctypes.c_int64, P, P],
            "moe_dispatch_noalloc": [cfgp, P, P, P, P, P, P, P, P, P, P],
            "moe_kernel_launches": [],
            "moe_backward_workspace_size": [cfgp, ctypes.POINTER(ctypes.c_size_t)],
            "moe_layer_backward": [cfgp, ctypes.c_float, ctypes.POINTER(moe_backward_io), P, P],
            "moe_expert_ffn_segments": [cfgp, P, P, P, P, ctypes.c_int32] + [P] * 9,
        }
        restype = {"moe_status_string": ctypes.c_char_p, "moe_kernel_launches": ctypes.c_uint64}
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = restype.get(name, I)
        _LIB = L
    return _LIB


def make_config(shape=None, **kw) -> moe_config:
    """moe_config from any object with the fields T, d_model, n_routed, top_k,
    d_ff, n_shared, d_ff_shared, capacity_factor, alpha, dtype, bias_mode,
    capacity_priority, overflow_mode (keyword arguments override)."""
    fields = [f for f, _ in moe_config._fields_]
    vals = {f: getattr(shape, f) for f in fields if shape is not None and hasattr(shape, f)}
    vals.update(kw)
    vals.setdefault("n_shared", 0)
    vals.setdefault("d_ff_shared", 0)
    vals.setdefault("capacity_factor", 0.0)
    vals.setdefault("alpha", 0.01)
    vals.setdefault("dtype", MOE_BF16)
    vals.setdefault("bias_mode", MOE_BIAS_LOGITS)
    vals.setdefault("capacity_priority", MOE_PRIORITY_TOKEN)
    vals.setdefault("overflow_mode", MOE_OVERFLOW_DROP)
    return moe_config(**{f: vals[f] for f in fields})


def _p(t) -> Optional[int]:
    """Device pointer of a tensor (None for None)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


def moe_workspace_size(cfg: moe_config) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def moe_buffer_rows(cfg: moe_config):
    """(capacity or -1, R_cap, x_disp rows, y rows)."""
    vals = [ctypes.c_int32(0) for _ in range(4)]
    _check(lib().moe_buffer_rows(ctypes.byref(cfg), *[ctypes.byref(v) for v in vals]), "moe_buffer_rows")
    return tuple(v.value for v in vals)


def moe_workspace_init(cfg, ws, stream=None):
    _check(lib().moe_workspace_init(ctypes.byref(cfg), _p(ws), _stream(stream)), "moe_workspace_init")


def moe_get_device_status(cfg, ws, stream=None, clear: bool = False) -> int:
    st = ctypes.c_int32(0)
    _check(lib().moe_get_device_status(ctypes.byref(cfg), _p(ws), _stream(stream), ctypes.byref(st),
                                       1 if clear else 0), "moe_get_device_status")
    return st.value


def moe_kernel_launches() -> int:
    """Kernels the library has launched in this process since it was loaded."""
    return int(lib().moe_kernel_launches())


def moe_route(cfg, x, W_r, logit_bias, topk_idx, gates, logits_out, ws, stream=None):
    _check(lib().moe_route(ctypes.byref(cfg), _p(x), _p(W_r), _p(logit_bias), _p(topk_idx), _p(gates),
                           _p(logits_out), _p(ws), _stream(stream)), "moe_route")


def moe_dispatch(cfg, x, topk_idx, counts, kept, offsets, slot_row, row_slot, x_disp, x_disp_scales,
                 ws, stream=None):
    _check(lib().moe_dispatch(ctypes.byref(cfg), _p(x), _p(topk_idx), _p(counts), _p(kept), _p(offsets),
                              _p(slot_row), _p(row_slot), _p(x_disp), _p(x_disp_scales), _p(ws),
                              _stream(stream)), "moe_dispatch")


def moe_expert_ffn(cfg, x, x_disp, x_disp_scales, offsets, W1, W1_scales, b1, W2, W2_scales, b2,
                   Ws1, Ws1_scales, bs1, Ws2, Ws2_scales, bs2, y, ws, stream=None):
    _check(lib().moe_expert_ffn(ctypes.byref(cfg), _p(x), _p(x_disp), _p(x_disp_scales), _p(offsets),
                                _p(W1), _p(W1_scales), _p(b1), _p(W2), _p(W2_scales), _p(b2),
                                _p(Ws1), _p(Ws1_scales), _p(bs1), _p(Ws2), _p(Ws2_scales), _p(bs2),
                                _p(y), _p(ws), _stream(stream)), "moe_expert_ffn")


def moe_expert_ffn_segments(cfg, x_rows, x_rows_scales, seg_offsets, seg_expert, n_seg: int,
                            W1, W1_scales, b1, W2, W2_scales, b2, y, ws, stream=None):
    """The grouped expert FFN over caller-made segments: rows seg_offsets[i] ..
    seg_offsets[i+1]-1 of x_rows through expert seg_expert[i] (cfg: the held
    experts, top_k 1, T = rows, no shared experts, no capacity)."""
    _check(lib().moe_expert_ffn_segments(ctypes.byref(cfg), _p(x_rows), _p(x_rows_scales), _p(seg_offsets),
                                         _p(seg_expert), int(n_seg), _p(W1), _p(W1_scales), _p(b1), _p(W2),
                                         _p(W2_scales), _p(b2), _p(y), _p(ws), _stream(stream)),
           "moe_expert_ffn_segments")


def moe_combine(cfg, y, gates, slot_row, out, stream=None, x=None):
    """x (the layer input) is read only with overflow_mode = MOE_OVERFLOW_PASS."""
    _check(lib().moe_combine(ctypes.byref(cfg), _p(y), _p(gates), _p(slot_row), _p(x), _p(out),
                             _stream(stream)), "moe_combine")


def moe_balance_stats(cfg, counts, ws, f, P, loss, stream=None):
    _check(lib().moe_balance_stats(ctypes.byref(cfg), _p(counts), _p(ws), _p(f), _p(P), _p(loss),
                                   _stream(stream)), "moe_balance_stats")


def moe_layer_forward(cfg, x, W_r, logit_bias, W1, W1_scales, b1, W2, W2_scales, b2,
                      Ws1, Ws1_scales, bs1, Ws2, Ws2_scales, bs2, out, f, P, loss,
                      topk_idx, gates, counts, ws, stream=None):
    _check(lib().moe_layer_forward(ctypes.byref(cfg), _p(x), _p(W_r), _p(logit_bias), _p(W1), _p(W1_scales),
                                   _p(b1), _p(W2), _p(W2_scales), _p(b2), _p(Ws1), _p(Ws1_scales), _p(bs1),
                                   _p(Ws2), _p(Ws2_scales), _p(bs2), _p(out), _p(f), _p(P), _p(loss),
                                   _p(topk_idx), _p(gates), _p(counts), _p(ws), _stream(stream)),
           "moe_layer_forward")


def moe_selftest_wait_timeout(cfg, timeout_ns: int, ws, stream=None):
    _check(lib().moe_selftest_wait_timeout(ctypes.byref(cfg), int(timeout_ns), _p(ws), _stream(stream)),
           "moe_selftest_wait_timeout")


def moe_backward_workspace_size(cfg: moe_config) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_backward_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "moe_backward_workspace_size")
    return n.value


def backward_io(tensors: dict) -> moe_backward_io:
    """moe_backward_io from a dict of tensors keyed by the header's field
    names (missing or None fields are NULL)."""
    unknown = set(tensors) - set(BACKWARD_IO_FIELDS)
    if unknown:
        raise KeyError(f"not moe_backward_io fields: {sorted(unknown)}")
    return moe_backward_io(**{n: _p(tensors.get(n)) for n in BACKWARD_IO_FIELDS})


def moe_layer_backward(cfg, lam: float, tensors: dict, bws, stream=None):
    """Gradients of <dout, out> + lam * L_balance (fp32, written into the dx,
    dW_r, ... tensors of `tensors`); bws: moe_backward_workspace_size() bytes."""
    io = backward_io(tensors)
    _check(lib().moe_layer_backward(ctypes.byref(cfg), ctypes.c_float(lam), ctypes.byref(io), _p(bws),
                                    _stream(stream)), "moe_layer_backward")


def moe_dispatch_noalloc(cfg, x, topk_idx, counts, kept, offsets, slot_row, row_slot, x_disp,
                         x_disp_scales, stream=None):
    """moe_dispatch with its scratch in the library's own 2 MiB device array
    instead of a workspace: for callers that cannot allocate device memory.
    Calls that overlap on the GPU race on that array."""
    _check(lib().moe_dispatch_noalloc(ctypes.byref(cfg), _p(x), _p(topk_idx), _p(counts), _p(kept),
                                      _p(offsets), _p(slot_row), _p(row_slot), _p(x_disp),
                                      _p(x_disp_scales), _stream(stream)), "moe_dispatch_noalloc")


class MoELayer:
    """A layer shape plus device-resident weights and workspace.

    weights: dict with W_r, logit_bias (or None), W1, W1_scales, b1, W2,
    W2_scales, b2, Ws1, Ws1_scales, bs1, Ws2, Ws2_scales, bs2 (CUDA tensors or
    None where not used).  forward(x) runs moe_layer_forward on the current
    stream and returns (out, f, P, loss).
    """

    def __init__(self, cfg: moe_config, weights: dict, device="cuda"):
        import torch
        self.cfg = cfg
        self.w = weights
        self.device = torch.device(device)
        self.ws = torch.empty(moe_workspace_size(cfg), dtype=torch.uint8, device=self.device)
        moe_workspace_init(cfg, self.ws)
        out_dt = torch.float32 if cfg.dtype == MOE_F32 else torch.bfloat16
        self.out = torch.empty((cfg.T, cfg.d_model), dtype=out_dt, device=self.device)
        self.f = torch.empty(cfg.n_routed, dtype=torch.float32, device=self.device)
        self.P = torch.empty(cfg.n_routed, dtype=torch.float32, device=self.device)
        self.loss = torch.empty(1, dtype=torch.float32, device=self.device)
        self.topk_idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device=self.device)
        self.gates = torch.empty((cfg.T, cfg.top_k), dtype=torch.float32, device=self.device)
        self.counts = torch.empty(cfg.n_routed, dtype=torch.int32, device=self.device)

    def forward(self, x, stream=None):
        w = self.w
        g = lambda k: w.get(k)  # noqa: E731
        moe_layer_forward(self.cfg, x, g("W_r"), g("logit_bias"), g("W1"), g("W1_scales"), g("b1"),
                          g("W2"), g("W2_scales"), g("b2"), g("Ws1"), g("Ws1_scales"), g("bs1"),
                          g("Ws2"), g("Ws2_scales"), g("bs2"), self.out, self.f, self.P, self.loss,
                          self.topk_idx, self.gates, self.counts, self.ws, stream)
        return self.out, self.f, self.P, self.loss

    def _forward_into(self, x, out, loss, stream=None):
        w = self.w
        g = lambda k: w.get(k)  # noqa: E731
        moe_layer_forward(self.cfg, x, g("W_r"), g("logit_bias"), g("W1"), g("W1_scales"), g("b1"),
                          g("W2"), g("W2_scales"), g("b2"), g("Ws1"), g("Ws1_scales"), g("bs1"),
                          g("Ws2"), g("Ws2_scales"), g("bs2"), out, self.f, self.P, loss,
                          self.topk_idx, self.gates, self.counts, self.ws, stream)

    def forward_host_batches(self, x_hosts, out_hosts, loss_hosts, between=None):
        """Runs the layer on consecutive batches that live in pinned host
        memory and writes each batch's output and loss back to host memory.

        Batch k's host->device copy runs on a copy-in stream and its
        device->host copies on a copy-out stream, so they overlap the compute
        of batches k-1 and k+1 (device inputs and outputs are double-buffered;
        events order the three streams).  `between`, if given, is called on
        the compute stream before each batch.  Returns the (start, end) CUDA
        events that bracket the whole run: the first input copy to the last
        output copy.  f, P, topk_idx, gates and counts hold the last batch's."""
        import torch
        dev = self.device
        n = len(x_hosts)
        assert len(out_hosts) == n and len(loss_hosts) == n
        cur = torch.cuda.current_stream(dev)
        s_in = torch.cuda.Stream(device=dev)
        s_out = torch.cuda.Stream(device=dev)
        x_dev = [torch.empty_like(x_hosts[0], device=dev) for _ in range(2)]
        out_dev = [torch.empty_like(self.out) for _ in range(2)]
        loss_dev = [torch.empty_like(self.loss) for _ in range(2)]
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready = [ev(), ev()]
        computed = [ev(), ev()]
        copied_out = [ev(), ev()]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_in.wait_stream(cur)
        s_out.wait_stream(cur)
        start.record(s_in)
        for k in range(n):
            b = k & 1
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(computed[b])            # x_dev[b] no longer read
                x_dev[b].copy_(x_hosts[k], non_blocking=True)
                in_ready[b].record(s_in)
            cur.wait_event(in_ready[b])
            if k >= 2:
                cur.wait_event(copied_out[b])               # out_dev[b] already copied back
            if between is not None:
                between()
            self._forward_into(x_dev[b], out_dev[b], loss_dev[b], stream=cur)
            computed[b].record(cur)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[b])
                out_hosts[k].copy_(out_dev[b], non_blocking=True)
                loss_hosts[k].copy_(loss_dev[b], non_blocking=True)
                copied_out[b].record(s_out)
        end.record(s_out)
        cur.wait_stream(s_out)
        return start, end

    def device_status(self, clear: bool = False) -> int:
        return moe_get_device_status(self.cfg, self.ws, clear=clear)

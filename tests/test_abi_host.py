"""Host-side checks of the C ABI: the library loads, exports every declared
entry point, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
import sparse_mixture_experts_20_b200 as M
from synthetic import DTYPE_F32, WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"MOE_EXPORT\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text))
    return names


def test_library_loads_and_exports_every_declared_symbol():
    L = M.lib()
    names = declared_symbols()
    assert len(names) >= 13
    for n in sorted(names):
        assert hasattr(L, n), n
    assert set(M.EXPORTED) <= names


def declared_arity():
    """Parameter count of every exported function in include/*.h."""
    out = {}
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            for m in re.finditer(r"MOE_EXPORT\s+[\w\s\*]+?\b(moe_\w+)\s*\(([^)]*)\)", text):
                params = [p for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
                out[m.group(1)] = len(params)
    return out


def test_binding_signatures_match_header():
    """The ctypes argument lists have exactly the header's parameter count
    (an extra argument would be passed as a C varargs int)."""
    L = M.lib()
    ar = declared_arity()
    for name, n in ar.items():
        assert len(getattr(L, name).argtypes) == n, (name, n, len(getattr(L, name).argtypes))


def test_status_strings():
    L = M.lib()
    assert L.moe_status_string(0) == b"MOE_OK"
    assert L.moe_status_string(5) == b"MOE_ERR_DEVICE_TIMEOUT"


@pytest.mark.parametrize("cid", sorted(WORKLOADS))
def test_workspace_and_rows_for_every_config(cid):
    sh = WORKLOADS[cid]
    cfg = M.make_config(sh)
    assert M.moe_workspace_size(cfg) > 0
    cap, r_cap, xr, yr = M.moe_buffer_rows(cfg)
    C = O.capacity_of(sh.T, sh.top_k, sh.n_routed, sh.capacity_factor)
    assert cap == (-1 if C is None else C)
    assert r_cap == (sh.T * sh.top_k if C is None else min(sh.T * sh.top_k, sh.n_routed * C))
    assert yr == r_cap + sh.n_shared * sh.T
    assert xr == r_cap + (sh.T if (sh.dtype == 2 and sh.n_shared) else 0)


def test_capacity_is_exact_ceiling():
    rng = np.random.default_rng(0)
    for _ in range(2000):
        T = int(rng.integers(1, 5000))
        E = int(rng.integers(1, 257))
        K = int(rng.integers(1, min(E, 16) + 1))
        cf = float(np.float32(rng.choice([rng.uniform(0.01, 3.0), 1.0, 1.25, 0.5, 2.0])))
        cfg = M.make_config(T=T, d_model=64, n_routed=E, top_k=K, d_ff=64, capacity_factor=cf)
        cap = M.moe_buffer_rows(cfg)[0]
        assert cap == O.capacity_of(T, K, E, cf), (T, E, K, cf)


@pytest.mark.parametrize("bad", [
    dict(T=0), dict(d_model=0), dict(n_routed=0), dict(top_k=0), dict(top_k=9), dict(d_ff=0),
    dict(n_shared=-1), dict(n_shared=1, d_ff_shared=0), dict(capacity_factor=-1.0),
    dict(capacity_factor=float("inf")), dict(dtype=7),
])
def test_invalid_config_rejected(bad):
    kw = dict(T=64, d_model=128, n_routed=8, top_k=2, d_ff=256)
    kw.update(bad)
    cfg = M.make_config(**kw)
    n = ctypes.c_size_t(0)
    assert M.lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == M.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [
    dict(n_routed=300), dict(top_k=17, n_routed=32), dict(n_shared=9, d_ff_shared=64),
    dict(d_model=96), dict(d_ff=200), dict(dtype=2, d_model=192), dict(dtype=2, d_ff=64),
])
def test_unsupported_shapes_rejected(bad):
    kw = dict(T=64, d_model=128, n_routed=8, top_k=2, d_ff=256)
    kw.update(bad)
    cfg = M.make_config(**kw)
    n = ctypes.c_size_t(0)
    assert M.lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == M.MOE_ERR_UNSUPPORTED


def test_null_pointers_rejected_without_launch():
    L = M.lib()
    launches_before = M.moe_kernel_launches()
    cfg = M.make_config(T=64, d_model=128, n_routed=8, top_k=2, d_ff=256)
    c = ctypes.byref(cfg)
    assert L.moe_route(c, None, None, None, None, None, None, None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_dispatch(c, *([None] * 11)) == M.MOE_ERR_INVALID_ARG
    assert L.moe_expert_ffn(c, *([None] * 19)) == M.MOE_ERR_INVALID_ARG
    assert L.moe_combine(c, None, None, None, None, None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_balance_stats(c, None, None, None, None, None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_layer_forward(c, *([None] * 24)) == M.MOE_ERR_INVALID_ARG
    # misaligned workspace / inputs (fake, never dereferenced)
    assert L.moe_route(c, 0x1000, 0x1000, None, 0x1000, 0x1000, None, 0x1001, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_route(c, 0x1008, 0x1000, None, 0x1000, 0x1000, None, 0x1000, None) == M.MOE_ERR_INVALID_ARG
    # every rejection happened on the host, before any kernel was launched
    assert M.moe_kernel_launches() == launches_before


def test_bias_mode_validated():
    cfg = M.make_config(T=64, d_model=128, n_routed=8, top_k=2, d_ff=256, bias_mode=2)
    n = ctypes.c_size_t(0)
    assert M.lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == M.MOE_ERR_INVALID_ARG
    cfg.bias_mode = M.MOE_BIAS_SELECTION
    assert M.lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == M.MOE_OK


def test_fp8_requires_scales():
    L = M.lib()
    cfg = M.make_config(T=64, d_model=128, n_routed=8, top_k=2, d_ff=128, dtype=2)
    p = 0x10000
    args = [p] * 8 + [None, p, None]     # x .. x_disp valid, x_disp_scales NULL, ws, stream
    assert L.moe_dispatch(ctypes.byref(cfg), *args) == M.MOE_ERR_INVALID_ARG


def _r256(n):
    return (n + 255) // 256 * 256


def _bwd_layout_bytes(T, d, E, K, dff, S, dffs, r_cap):
    """Closed form of the fp32 layers' backward scratch: fp32 regions, each
    rounded up to 256 bytes, in the order status, a, dl, dy, z, dz, dx rows,
    shared dy, z, dz, dx."""
    regions = [64, T * K, T * E, r_cap * d, r_cap * dff, r_cap * dff, r_cap * d,
               T * d if S else 0, T * dffs if S else 0, T * dffs if S else 0, T * d]
    return sum(_r256(n * 4) for n in regions)


def _bwd_tc_layout_bytes(T, d, E, K, dff, S, dffs, r_cap):
    """Closed form of the bf16 layers' backward scratch: status word; fp32 a,
    dl; bf16 dl (row stride N_r rounded up to 8) and W_r; fp32 partials of the
    router weight gradient when its tokens are split (about 296 output tiles
    at once, at most one split per 256 tokens, chunks of a multiple of 16
    tokens); fp32 router dx; padded row offsets; routed rows padded to 16 per
    expert (r_cap + 15 N_r, rounded to 16): bf16 x, dy, SiLU(z), SiLU'(z), dz
    and dx rows; shared bf16 SiLU(z), SiLU'(z), dz of width n_shared *
    d_ff_shared and fp32 dx; fp32 column-sum partials (16-row chunks of the
    routed rows and of the tokens)."""
    rp = (r_cap + 15 * E + 15) // 16 * 16
    sw = S * dffs
    epad = (E + 7) // 8 * 8
    tiles = ((E + 127) // 128) * ((d + 255) // 256)
    splits = min(-(-296 // tiles), (T + 255) // 256)
    splits = max(splits, 1)
    chunk = (-(-T // splits) + 15) // 16 * 16
    splits = -(-T // chunk)
    nch = (T + 15) // 16
    part = max((rp // 16) * max(d, dff), nch * max(d, sw), nch * E)
    regions = [256, T * K * 4, T * E * 4, T * epad * 2, E * d * 2, splits * E * d * 4 if splits > 1 else 0,
               T * d * 4, (E + 1) * 4,
               rp * d * 2, rp * d * 2, rp * dff * 2, rp * dff * 2, rp * dff * 2, rp * d * 2,
               T * sw * 2, T * sw * 2, T * sw * 2, T * d * 4 if sw else 0, part * 4]
    return sum(_r256(n) for n in regions)


@pytest.mark.parametrize("cid", [1, 2, 3])
def test_backward_workspace_closed_form(cid):
    sh = WORKLOADS[cid]
    cfg = M.make_config(sh)
    _, r_cap, _, _ = M.moe_buffer_rows(cfg)
    form = _bwd_layout_bytes if sh.dtype == DTYPE_F32 else _bwd_tc_layout_bytes
    assert M.moe_backward_workspace_size(cfg) == form(
        sh.T, sh.d_model, sh.n_routed, sh.top_k, sh.d_ff, sh.n_shared, sh.d_ff_shared, r_cap)


def test_backward_rejects_fp8_and_bad_arguments_without_launch():
    L = M.lib()
    before = M.moe_kernel_launches()
    n = ctypes.c_size_t(0)
    fp8 = M.make_config(WORKLOADS[4])
    assert L.moe_backward_workspace_size(ctypes.byref(fp8), ctypes.byref(n)) == M.MOE_ERR_UNSUPPORTED
    io = M.moe_backward_io()
    assert L.moe_layer_backward(ctypes.byref(fp8), 1.0, ctypes.byref(io), 0x1000, None) == M.MOE_ERR_UNSUPPORTED
    cfg = M.make_config(T=64, d_model=128, n_routed=8, top_k=2, d_ff=128, n_shared=1, d_ff_shared=64)
    c = ctypes.byref(cfg)
    assert L.moe_layer_backward(c, 1.0, None, 0x1000, None) == M.MOE_ERR_INVALID_ARG
    # every field set to an aligned fake address except one required pointer:
    # rejected on the host (the fakes are never dereferenced)
    fake = {f: 0x10000 for f in M.BACKWARD_IO_FIELDS}
    for missing in ("x", "logits", "row_slot", "dout", "dx", "dW1", "dWs2"):
        io = M.moe_backward_io(**{k: (None if k == missing else v) for k, v in fake.items()})
        assert L.moe_layer_backward(c, 1.0, ctypes.byref(io), 0x1000, None) == M.MOE_ERR_INVALID_ARG, missing
    io = M.moe_backward_io(**{k: (0x10008 if k == "y" else v) for k, v in fake.items()})
    assert L.moe_layer_backward(c, 1.0, ctypes.byref(io), 0x1000, None) == M.MOE_ERR_INVALID_ARG
    io = M.moe_backward_io(**{k: (None if k == "dx" else v) for k, v in fake.items()})
    assert L.moe_layer_backward(c, float("nan"), ctypes.byref(io), 0x1000, None) == M.MOE_ERR_INVALID_ARG
    assert M.moe_kernel_launches() == before


def test_backward_io_binding_names_every_field():
    assert M.BACKWARD_IO_FIELDS[0] == "x" and M.BACKWARD_IO_FIELDS[-1] == "dbs2"
    assert len(M.BACKWARD_IO_FIELDS) == 31
    hdr = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    body = hdr[hdr.index("typedef struct moe_backward_io"):hdr.index("} moe_backward_io;")]
    declared = re.findall(r"\*\s*(\w+);", body)
    assert tuple(declared) == M.BACKWARD_IO_FIELDS
    with pytest.raises(KeyError):
        M.backward_io({"not_a_field": None})


def test_expert_ffn_segments_rejects_bad_arguments_without_launch():
    """moe_expert_ffn_segments: a layer with shared experts, top_k != 1, a
    capacity, no segments or more than 256, a missing segment map or missing
    FP8 scales are argument errors caught on the host (the fake addresses are
    never dereferenced)."""
    L = M.lib()
    before = M.moe_kernel_launches()
    p, ws = 0x10000, 0x100000

    def call(cfg, n_seg=4, seg_expert=p, scales=None):
        return L.moe_expert_ffn_segments(ctypes.byref(cfg), p, scales, p, seg_expert, n_seg, p, scales, p, p,
                                         scales, p, p, ws, None)

    base = dict(T=64, d_model=128, n_routed=4, top_k=1, d_ff=128)
    ok = M.make_config(**base)
    for bad in (dict(n_seg=0), dict(n_seg=257), dict(seg_expert=None), dict(seg_expert=p + 4)):
        assert call(ok, **bad) == M.MOE_ERR_INVALID_ARG, bad
    assert call(M.make_config(**dict(base, n_shared=1, d_ff_shared=64))) == M.MOE_ERR_INVALID_ARG
    assert call(M.make_config(**dict(base, top_k=2))) == M.MOE_ERR_INVALID_ARG
    assert call(M.make_config(**dict(base, capacity_factor=1.0))) == M.MOE_ERR_INVALID_ARG
    fp8 = M.make_config(**dict(base, d_model=128, d_ff=256, dtype=M.MOE_FP8_E4M3_BLOCK))
    assert call(fp8) == M.MOE_ERR_INVALID_ARG                 # FP8 rows without their scales
    assert M.moe_kernel_launches() == before

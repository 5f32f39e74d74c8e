"""PISA piecewise sparse attention for NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/pisa.h`` (``libpisa.so``,
built in-tree by ``python -m block_sparse_attention_pisa_b200.build``). The
binding only marshals arguments: it reads shapes and device pointers from
torch tensors, allocates outputs with torch, and passes torch's current CUDA
stream. Every step of the computation runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback -- if the library is missing or the
device is not a B200 the calls raise.

Method: "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
Transformers" (explainer of arXiv 2602.01077 on gist.science), technical
summary section 2.
"""
from __future__ import annotations

import ctypes
import os

ORDER_DROP, ORDER_ZERO, ORDER_FIRST, ORDER_HYBRID = -1, 0, 1, 2

__all__ = [
    "ORDER_DROP", "ORDER_ZERO", "ORDER_FIRST", "ORDER_HYBRID", "PisaError", "Shape", "HostOptions", "lib", "block_stats", "select", "attention", "attention_simt",
    "pisa", "pisa_host", "pisa_host_static", "STATIC_WORKSPACE_BYTES", "host_workspace_bytes", "head_chunks", "device_error", "num_blocks", "LIB_PATH", "SYMBOLS", "routing_norms",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpisa.so")

# entry points declared in include/pisa.h
SYMBOLS = (
    "pisa_block_stats", "pisa_select", "pisa_routing_norms", "pisa_attention", "pisa_attention_simt",
    "pisa_device_error", "pisa_status_string", "pisa_last_error", "pisa_version",
    "pisa_run_host_workspace", "pisa_run_host", "pisa_select_grouped", "pisa_run_host_static",
)

# PISA_STATIC_WORKSPACE_BYTES in include/pisa.h: the device region pisa_run_host_static uses
STATIC_WORKSPACE_BYTES = 32 << 20

STATUS = {0: "PISA_OK", 1: "PISA_ERR_INVALID_ARG", 2: "PISA_ERR_UNSUPPORTED",
          3: "PISA_ERR_CUDA", 4: "PISA_ERR_TIMEOUT"}


class PisaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("block", ctypes.c_int32)]


class HostOptions(ctypes.Structure):
    """pisa_host_options_t: routing weight, grouped selection and pipeline ranges (0: default)."""
    _fields_ = [("route_lambda", ctypes.c_float), ("group", ctypes.c_int32),
                ("candidates", ctypes.c_int32), ("chunks", ctypes.c_int32)]


_lib = None


def lib():
    """The loaded ``libpisa.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_pisa_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    L.pisa_block_stats.argtypes = [vp, vp, Shape, i32, vp, vp, vp, vp]
    L.pisa_select.argtypes = [vp, vp, vp, f32, Shape, i32, vp, vp]
    L.pisa_select_grouped.argtypes = [vp, vp, vp, f32, Shape, i32, i32, i32, vp, vp]
    L.pisa_routing_norms.argtypes = [vp, Shape, vp, vp, vp]
    attn = [vp, vp, vp, vp, vp, vp, vp, Shape, i32, i32, f32, vp, vp]
    L.pisa_attention.argtypes = attn
    L.pisa_attention_simt.argtypes = attn
    opts = ctypes.POINTER(HostOptions)
    L.pisa_run_host_workspace.argtypes = [Shape, i32, i32, opts, ctypes.POINTER(ctypes.c_size_t)]
    L.pisa_run_host.argtypes = [vp, vp, vp, Shape, i32, i32, f32, opts, vp, ctypes.c_size_t, vp, vp]
    L.pisa_run_host_static.argtypes = [vp, vp, vp, Shape, i32, i32, f32, opts, vp, vp]
    L.pisa_device_error.argtypes = [vp]
    L.pisa_status_string.argtypes = [ctypes.c_int]
    L.pisa_status_string.restype = ctypes.c_char_p
    L.pisa_last_error.argtypes = []
    L.pisa_last_error.restype = ctypes.c_char_p
    L.pisa_version.argtypes = []
    for name in ("pisa_block_stats", "pisa_select", "pisa_routing_norms", "pisa_attention", "pisa_attention_simt",
                 "pisa_device_error", "pisa_version", "pisa_run_host_workspace", "pisa_run_host",
                 "pisa_select_grouped", "pisa_run_host_static"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(status: int):
    if status != 0:
        raise PisaError(status, lib().pisa_last_error().decode())


def num_blocks(N: int, block: int) -> int:
    return -(-N // block)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _shape(x, block: int) -> Shape:
    if x.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    if not x.is_contiguous():
        raise ValueError("tensors must be contiguous [B, H, N, d]")
    B, H, N, d = x.shape
    return Shape(B, H, N, d, block)


def _require(t, name: str, shape, dtype, device=None):
    """Raise ValueError unless ``t`` is a contiguous tensor of exactly ``shape`` and
    ``dtype`` (and, when ``device`` is given, on that CUDA device). Shapes and dtypes
    are checked first, so a wrong buffer is named before any device question."""
    import torch
    if t is None:
        raise ValueError(f"{name} is required here")
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch tensor")
    if tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(int(x) for x in shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _device_of(t):
    """The CUDA device of the operands (``t`` must live on one)."""
    if not t.is_cuda:
        raise ValueError("the operands must be CUDA tensors")
    return t.device


def _stat_shapes(s: Shape, order: int):
    """(kbar / S0 shape, first-order statistic shape or None) for one order."""
    nB = num_blocks(s.N, s.block)
    kb = (s.B, s.H, nB, s.d)
    if order == ORDER_FIRST:
        return kb, (s.B, s.H, nB, s.d, s.d)
    if order == ORDER_HYBRID:
        return kb, (s.B, s.H, s.d, s.d)
    return kb, None


def _first_order_dtype(order: int):
    import torch
    return torch.bfloat16 if order == ORDER_FIRST else torch.float32


def _check_order(order: int):
    if order not in (ORDER_DROP, ORDER_ZERO, ORDER_FIRST, ORDER_HYBRID):
        raise ValueError(f"order={order} (must be -1, 0, 1 or 2)")


def block_stats(K, V, block: int, order: int = 1, out=None):
    """kbar (fp32), S0 (fp32) and the first-order statistic of every key/value block:
    per-block S1 (bf16 [B, H, nB, d, d]) at order 1, the head's Hbar (fp32
    [B, H, d, d]) at order 2, None at orders 0 and -1.
    ``out`` = (kbar, S0, S1) preallocated outputs (optional)."""
    import torch
    s = _shape(K, block)
    _check_order(order)
    nB = num_blocks(s.N, block)
    kb_shape, s1_shape = _stat_shapes(s, order)
    _require(K, "K", K.shape, torch.bfloat16)
    _require(V, "V", K.shape, torch.bfloat16)
    outs = []
    if out is not None:
        kbar, S0, S1 = out
        outs = [(kbar, "kbar", kb_shape, torch.float32), (S0, "S0", kb_shape, torch.float32)]
        if s1_shape is not None:
            outs.append((S1, "S1", s1_shape, _first_order_dtype(order)))
        else:
            S1 = None
        for t, name, shp, dt in outs:
            _require(t, name, shp, dt)
    dev = _device_of(K)
    for t, name in [(V, "V")] + [(x, n) for x, n, _, _ in outs]:
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}")
    if out is None:
        kbar = torch.empty((s.B, s.H, nB, s.d), device=K.device, dtype=torch.float32)
        S0 = torch.empty_like(kbar)
        S1 = torch.empty(s1_shape, device=K.device, dtype=_first_order_dtype(order)) if s1_shape else None
    _check(lib().pisa_block_stats(_ptr(K), _ptr(V), s, order, _ptr(kbar), _ptr(S0), _ptr(S1),
                                  _stream(K)))
    return kbar, S0, S1


def select(Q, kbar, block: int, topk: int, out=None, route=None, lam: float = 0.0,
           group: int = 1, candidates: int | None = None):
    """int32 [B, H, nB, topk]: critical blocks of every query block (ascending).
    ``route`` (fp32 [B, H, nB], from ``routing_norms``) and ``lam`` add the
    covariance term lam * M_j to every score. With ``group`` > 1 (or ``candidates``
    below nB) the selection is grouped: one proxy query per ``group`` query blocks keeps
    ``candidates`` key blocks, and each member keeps its best ``topk`` of them
    (``candidates`` = topk hands the proxy's list to every member)."""
    import torch
    s = _shape(Q, block)
    nB = num_blocks(s.N, block)
    _require(Q, "Q", Q.shape, torch.bfloat16)
    _require(kbar, "kbar", (s.B, s.H, nB, s.d), torch.float32)
    if route is not None:
        _require(route, "route", (s.B, s.H, nB), torch.float32)
    if out is not None:
        _require(out, "idx", (s.B, s.H, nB, topk), torch.int32)
    dev = _device_of(Q)
    for t, name in ((kbar, "kbar"), (route, "route"), (out, "idx")):
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}")
    idx = (torch.empty((s.B, s.H, nB, topk), device=Q.device, dtype=torch.int32)
           if out is None else out)
    if group == 1 and (candidates is None or candidates == nB):
        _check(lib().pisa_select(_ptr(Q), _ptr(kbar), _ptr(route), float(lam), s, topk, _ptr(idx),
                                 _stream(Q)))
    else:
        cand = nB if candidates is None else int(candidates)
        _check(lib().pisa_select_grouped(_ptr(Q), _ptr(kbar), _ptr(route), float(lam), s, topk, int(group),
                                         cand, _ptr(idx), _stream(Q)))
    return idx


def routing_norms(S1, block: int, N: int, out=None):
    """(Hbar fp32 [B, H, d, d], M fp32 [B, H, nB]) from per-block bf16 S1 [B, H, nB, d, d]:
    the mean first-order matrix and each block's Frobenius deviation from it."""
    import torch
    if S1.dim() != 5 or S1.shape[-1] != S1.shape[-2]:
        raise ValueError("S1 must be [B, H, nB, d, d]")
    B, H, nB, d, _ = S1.shape
    if nB != num_blocks(N, block):
        raise ValueError("S1 block count does not match N and block")
    _require(S1, "S1", S1.shape, torch.bfloat16)
    s = Shape(B, H, N, d, block)
    if out is not None:
        Hbar, M = out
        _require(Hbar, "Hbar", (B, H, d, d), torch.float32)
        _require(M, "M", (B, H, nB), torch.float32)
    dev = _device_of(S1)
    if out is not None:
        for t, name in ((Hbar, "Hbar"), (M, "M")):
            if t.device != dev:
                raise ValueError(f"{name} is on {t.device}, expected {dev}")
    else:
        Hbar = torch.empty((B, H, d, d), device=S1.device, dtype=torch.float32)
        M = torch.empty((B, H, nB), device=S1.device, dtype=torch.float32)
    _check(lib().pisa_routing_norms(_ptr(S1), s, _ptr(Hbar), _ptr(M), _stream(S1)))
    return Hbar, M


def _attention(fn, Q, K, V, kbar, S0, S1, idx, block, order, scale, out=None):
    import torch
    s = _shape(Q, block)
    _check_order(order)
    nB = num_blocks(s.N, block)
    if idx is None or idx.dim() != 4:
        raise ValueError("idx must be an int32 [B, H, nB, topk] tensor")
    topk = int(idx.shape[-1])
    kb_shape, s1_shape = _stat_shapes(s, order)
    checks = [(Q, "Q", Q.shape, torch.bfloat16), (K, "K", Q.shape, torch.bfloat16),
              (V, "V", Q.shape, torch.bfloat16), (idx, "idx", (s.B, s.H, nB, topk), torch.int32)]
    if out is not None:
        checks.append((out, "O", Q.shape, torch.bfloat16))
    if order != ORDER_DROP:
        checks += [(kbar, "kbar", kb_shape, torch.float32), (S0, "S0", kb_shape, torch.float32)]
    if s1_shape is not None:
        checks.append((S1, "S1" if order == ORDER_FIRST else "Hbar (S1)", s1_shape, _first_order_dtype(order)))
    for t, name, shp, dt in checks:
        _require(t, name, shp, dt)
    dev = _device_of(Q)
    for t, name, _, _ in checks:
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}")
    if order == ORDER_DROP:
        kbar = S0 = S1 = None
    elif s1_shape is None:
        S1 = None
    O = torch.empty_like(Q) if out is None else out
    _check(fn(_ptr(Q), _ptr(K), _ptr(V), _ptr(kbar), _ptr(S0), _ptr(S1), _ptr(idx), s, topk,
              order, float(scale), _ptr(O), _stream(Q)))
    return O


def attention(Q, K, V, kbar, S0, S1, idx, block: int, order: int, scale: float, out=None):
    """Fused exact + Taylor attention; bf16 [B, H, N, d]. ``order``: -1 keep-or-drop,
    0 zeroth order, 1 per-block first order (S1 per block), 2 hybrid order (S1 = Hbar)."""
    return _attention(lib().pisa_attention, Q, K, V, kbar, S0, S1, idx, block, order, scale, out)


def attention_simt(Q, K, V, kbar, S0, S1, idx, block: int, order: int, scale: float, out=None):
    """The same operation on the plain CUDA-core cross-check kernel."""
    return _attention(lib().pisa_attention_simt, Q, K, V, kbar, S0, S1, idx, block, order, scale, out)


def pisa(Q, K, V, block: int, topk: int, order: int = 1, scale: float | None = None,
         route_lambda: float = 0.0, out=None, group: int = 1, candidates: int | None = None):
    """The whole path on device tensors: stats -> select -> attention. Returns (O, idx).
    With ``route_lambda`` > 0 the selection is covariance-aware: stats at order 1 ->
    routing norms -> routed select -> attention (at order 2 with the routing call's
    Hbar). ``group`` / ``candidates`` select with grouped proxies (see ``select``)."""
    if scale is None:
        scale = Q.shape[-1] ** -0.5
    sel = dict(group=group, candidates=candidates)
    if route_lambda > 0.0:
        kbar, S0, S1 = block_stats(K, V, block, ORDER_FIRST)
        Hbar, M = routing_norms(S1, block, Q.shape[2])
        idx = select(Q, kbar, block, topk, route=M, lam=route_lambda, **sel)
        first = Hbar if order == ORDER_HYBRID else (S1 if order == ORDER_FIRST else None)
        return attention(Q, K, V, kbar, S0, first, idx, block, order, scale, out=out), idx
    kbar, S0, S1 = block_stats(K, V, block, order)
    idx = select(Q, kbar, block, topk, **sel)
    return attention(Q, K, V, kbar, S0, S1, idx, block, order, scale, out=out), idx


def head_chunks(BH: int, chunks: int):
    """Split the flattened (batch, head) axis into `chunks` contiguous ranges of near-equal size."""
    chunks = max(1, min(chunks, BH))
    edges = [BH * c // chunks for c in range(chunks + 1)]
    return [(edges[c], edges[c + 1]) for c in range(chunks) if edges[c + 1] > edges[c]]


def host_workspace_bytes(shape: Shape, topk: int, order: int, route_lambda: float = 0.0, chunks: int = 0,
                         group: int = 1, candidates: int = 0) -> int:
    """Device workspace (bytes) that ``pisa_host`` needs for this problem."""
    n = ctypes.c_size_t(0)
    o = HostOptions(float(route_lambda), int(group), int(candidates), int(chunks))
    _check(lib().pisa_run_host_workspace(shape, int(topk), int(order), ctypes.byref(o), ctypes.byref(n)))
    return int(n.value)


def pisa_host(Q, K, V, block: int, topk: int, order: int = 1, scale: float | None = None,
              device="cuda", route_lambda: float = 0.0, chunks: int = 0, out=None,
              group: int = 1, candidates: int = 0):
    """The whole path on HOST tensors [B, H, N, d] through the C ABI's ``pisa_run_host``:
    the library copies Q, K, V to the device, runs the path and copies O back, pipelined
    over ``chunks`` ranges of (batch, head) pairs (copies of one range overlap the kernels
    of another; the result equals the whole-batch device path bit for bit). Pinned host
    tensors let the copies run asynchronously. ``group`` / ``candidates`` select with
    grouped proxies as ``select`` does. Returns O on the host (``out`` if given). The
    device workspace is allocated here with torch."""
    import torch
    if scale is None:
        scale = Q.shape[-1] ** -0.5
    s = _shape(Q, block)
    for t, name in ((Q, "Q"), (K, "K"), (V, "V")):
        _require(t, name, Q.shape, torch.bfloat16)
        if t.is_cuda:
            raise ValueError(f"{name} must be a host tensor (pisa_host copies it to the device)")
    if out is None:
        out = torch.empty(Q.shape, dtype=Q.dtype, pin_memory=Q.is_pinned())
    _require(out, "O", Q.shape, torch.bfloat16)
    if out.is_cuda:
        raise ValueError("O must be a host tensor")
    dev = torch.device(device)
    if dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    o = HostOptions(float(route_lambda), int(group), int(candidates or 0), int(chunks))
    with torch.cuda.device(dev):
        nbytes = ctypes.c_size_t(0)
        _check(lib().pisa_run_host_workspace(s, int(topk), int(order), ctypes.byref(o), ctypes.byref(nbytes)))
        ws = torch.empty(max(nbytes.value, 1), dtype=torch.uint8, device=dev)
        stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
        _check(lib().pisa_run_host(_ptr(Q), _ptr(K), _ptr(V), s, int(topk), int(order), float(scale),
                                   ctypes.byref(o), _ptr(ws), nbytes.value, _ptr(out), stream))
    return out


def pisa_host_static(Q, K, V, block: int, topk: int, order: int = 1, scale: float | None = None,
                     device="cuda", route_lambda: float = 0.0, chunks: int = 0, out=None,
                     group: int = 1, candidates: int = 0):
    """``pisa_host`` through the C ABI's ``pisa_run_host_static``: the device workspace is
    the library's fixed region (``STATIC_WORKSPACE_BYTES`` per device) and nothing is
    allocated on the device. Calls that overlap in time on one device race on that region.
    Returns O on the host (``out`` if given, else a new host tensor)."""
    import torch
    if scale is None:
        scale = Q.shape[-1] ** -0.5
    s = _shape(Q, block)
    for t, name in ((Q, "Q"), (K, "K"), (V, "V")):
        _require(t, name, Q.shape, torch.bfloat16)
        if t.is_cuda:
            raise ValueError(f"{name} must be a host tensor (pisa_host_static copies it to the device)")
    if out is None:
        out = torch.empty(Q.shape, dtype=Q.dtype, pin_memory=Q.is_pinned())
    _require(out, "O", Q.shape, torch.bfloat16)
    if out.is_cuda:
        raise ValueError("O must be a host tensor")
    dev = torch.device(device)
    if dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    o = HostOptions(float(route_lambda), int(group), int(candidates or 0), int(chunks))
    with torch.cuda.device(dev):
        stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
        _check(lib().pisa_run_host_static(_ptr(Q), _ptr(K), _ptr(V), s, int(topk), int(order), float(scale),
                                          ctypes.byref(o), _ptr(out), stream))
    return out


def device_error(stream_tensor=None):
    """Synchronise the current stream and raise if a kernel flagged the device error word."""
    import torch
    st = torch.cuda.current_stream().cuda_stream if stream_tensor is None else _stream(stream_tensor).value
    _check(lib().pisa_device_error(ctypes.c_void_p(st)))

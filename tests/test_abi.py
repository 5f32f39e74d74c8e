"""The C-ABI library on the CPU: it loads, exports every entry point that
include/pisa.h declares, and rejects bad arguments on the host before any
launch. Nothing here launches a kernel."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_pisa_b200 as P
from block_sparse_attention_pisa_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pisa.h")

OK, INVALID, UNSUPPORTED, CUDA_ERR = 0, 1, 2, 3
FAKE = 0x7f0000100000          # 16-byte aligned, never dereferenced (validation stops first)
MISALIGNED = FAKE + 4


@pytest.fixture(scope="module")
def L():
    B.build()
    return P.lib()


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\S.*?\b(pisa_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_binding_symbols():
    assert _declared() == sorted(P.SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in range(5):
        assert L.pisa_status_string(code)
    assert L.pisa_version() >= 100


def shape(B=1, H=2, N=256, d=128, block=64):
    return P.Shape(B, H, N, d, block)


def vp(x):
    return ctypes.c_void_p(x)


def stats(L, s=None, K=FAKE, V=FAKE, order=1, kbar=FAKE, S0=FAKE, S1=FAKE):
    return L.pisa_block_stats(vp(K), vp(V), s or shape(), order, vp(kbar), vp(S0), vp(S1), None)


def sel(L, s=None, Q=FAKE, kbar=FAKE, topk=2, idx=FAKE, route=0, lam=0.0):
    return L.pisa_select(vp(Q), vp(kbar), vp(route), lam, s or shape(), topk, vp(idx), None)


def attn(L, s=None, topk=2, order=1, scale=0.125, fn="pisa_attention", **ptrs):
    p = {k: FAKE for k in ("Q", "K", "V", "kbar", "S0", "S1", "idx", "O")}
    p.update(ptrs)
    return getattr(L, fn)(vp(p["Q"]), vp(p["K"]), vp(p["V"]), vp(p["kbar"]), vp(p["S0"]),
                          vp(p["S1"]), vp(p["idx"]), s or shape(), topk, order, scale,
                          vp(p["O"]), None)


def test_null_and_misaligned_pointers(L):
    assert stats(L, K=0) == INVALID
    assert b"K is NULL" in L.pisa_last_error()
    assert stats(L, V=MISALIGNED) == INVALID
    assert b"16-byte" in L.pisa_last_error()
    assert stats(L, S1=0) == INVALID            # order 1 needs S1
    assert sel(L, idx=0) == INVALID
    for name in ("Q", "K", "V", "kbar", "S0", "S1", "idx", "O"):
        assert attn(L, **{name: 0}) == INVALID, name
        assert attn(L, **{name: MISALIGNED}) == INVALID, name
        assert attn(L, fn="pisa_attention_simt", **{name: 0}) == INVALID, name


def test_bad_scalars(L):
    assert stats(L, order=3) == INVALID
    assert stats(L, order=-2) == INVALID
    assert sel(L, topk=0) == INVALID
    assert sel(L, topk=5) == INVALID            # nB = 4
    assert attn(L, topk=0) == INVALID
    assert attn(L, order=3) == INVALID
    assert attn(L, order=-2) == INVALID
    for sc in (0.0, -1.0, float("nan"), float("inf")):
        assert attn(L, scale=sc) == INVALID, sc
    assert attn(L, s=shape(N=-1)) == INVALID
    assert attn(L, s=shape(d=0)) == INVALID


def test_unsupported_shapes(L):
    assert stats(L, s=shape(d=96)) == UNSUPPORTED
    assert stats(L, s=shape(block=32)) == UNSUPPORTED
    assert sel(L, s=shape(N=64 * 2049), topk=4) == UNSUPPORTED   # nB > PISA_MAX_BLOCKS
    assert attn(L, s=shape(B=300, H=300)) == UNSUPPORTED


def _no_device():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("fake pointers must never reach a real device")


def _passes_validation(st, L):
    # validation passed: only the device check (no GPU here) remains
    assert st == CUDA_ERR, L.pisa_last_error()
    assert b"cuda" in L.pisa_last_error().lower()


def test_order0_needs_no_S1(L):
    _no_device()
    _passes_validation(stats(L, order=0, S1=0), L)
    _passes_validation(attn(L, order=0, S1=0), L)


def test_hybrid_order_needs_hbar(L):
    assert stats(L, order=2, S1=0) == INVALID
    assert b"Hbar" in L.pisa_last_error()
    assert attn(L, order=2, S1=0) == INVALID
    assert attn(L, order=2, S1=MISALIGNED) == INVALID
    _no_device()
    _passes_validation(stats(L, order=2), L)
    _passes_validation(attn(L, order=2), L)


def routing(L, s=None, S1=FAKE, Hbar=FAKE, M=FAKE):
    return L.pisa_routing_norms(vp(S1), s or shape(), vp(Hbar), vp(M), None)


def test_routing_arguments(L):
    for name in ("S1", "Hbar", "M"):
        assert routing(L, **{name: 0}) == INVALID, name
        assert routing(L, **{name: MISALIGNED}) == INVALID, name
    assert routing(L, s=shape(d=96)) == UNSUPPORTED
    assert routing(L, s=shape(N=0), S1=0, Hbar=0, M=0) == OK
    assert sel(L, route=MISALIGNED, lam=1.0) == INVALID
    for lam in (-1.0, float("nan"), float("inf")):
        assert sel(L, route=FAKE, lam=lam) == INVALID, lam
    _no_device()
    _passes_validation(routing(L), L)
    _passes_validation(sel(L, route=FAKE, lam=0.5), L)
    _passes_validation(sel(L, lam=-1.0), L)      # lambda is ignored without a route


def test_drop_needs_no_statistics(L):
    # keep-or-drop reads no kbar, S0 or S1 in the attention call
    assert attn(L, order=-1, idx=0) == INVALID
    _no_device()
    _passes_validation(attn(L, order=-1, kbar=0, S0=0, S1=0), L)
    _passes_validation(attn(L, order=-1, kbar=0, S0=0, S1=0, fn="pisa_attention_simt"), L)
    _passes_validation(stats(L, order=-1, S1=0), L)


def test_empty_problem_touches_nothing(L):
    # B*H*N == 0: OK with NULL pointers, no launch
    assert stats(L, s=shape(N=0), K=0, V=0, kbar=0, S0=0, S1=0) == OK
    assert sel(L, s=shape(H=0), Q=0, kbar=0, idx=0, topk=0) == OK
    assert attn(L, s=shape(B=0), Q=0, K=0, V=0, kbar=0, S0=0, S1=0, idx=0, O=0) == OK


def test_valid_call_without_gpu_reports_cuda_error(L):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("fake pointers must never reach a real device")
    assert stats(L) == CUDA_ERR
    assert sel(L) == CUDA_ERR
    assert attn(L) == CUDA_ERR


def test_binding_raises_on_missing_library(tmp_path, monkeypatch):
    monkeypatch.setattr(P, "LIB_PATH", str(tmp_path / "libpisa.so"))
    monkeypatch.setattr(P, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        P.lib()


def _opts(lam=0.0, chunks=8, group=1, cand=0):
    return ctypes.byref(P.HostOptions(lam, group, cand, chunks))


def _ws(L, s=None, topk=2, order=1, lam=0.0, chunks=8, group=1, cand=0):
    n = ctypes.c_size_t(123)
    st = L.pisa_run_host_workspace(s or shape(), topk, order, _opts(lam, chunks, group, cand), ctypes.byref(n))
    return st, n.value


def test_host_workspace_size(L):
    """3 slots of ceil(B*H / chunks) pairs: Q, K, V, O, kbar, S0, S1 (or Hbar), routing
    buffers and idx, each rounded up to 256 bytes."""
    up = lambda x: -(-x // 256) * 256  # noqa: E731
    B, H, N, d, b, k = 1, 24, 32768, 128, 64, 64
    nB = N // b
    R = 3                               # 24 pairs in 8 chunks
    act = up(R * N * d * 2)
    common = 4 * act + 2 * up(R * nB * d * 4) + up(R * nB * k * 4)
    st, n1 = _ws(L, shape(B, H, N, d, b), k, 1)
    assert st == OK and n1 == 3 * (common + up(R * nB * d * d * 2))
    st, n2 = _ws(L, shape(B, H, N, d, b), k, 2)
    assert st == OK and n2 == 3 * (common + up(R * d * d * 4))
    st, nr = _ws(L, shape(B, H, N, d, b), k, 2, lam=0.01)
    assert st == OK and nr == 3 * (common + up(R * nB * d * d * 2) + up(R * d * d * 4) + up(R * nB * 4))
    st, n0 = _ws(L, shape(B, H, N, d, b), k, -1, chunks=1)
    assert st == OK and n0 == 4 * up(24 * N * d * 2) + 2 * up(24 * nB * d * 4) + up(24 * nB * k * 4)
    assert _ws(L, shape(N=0)) == (OK, 0)
    assert _ws(L, chunks=-1)[0] == INVALID
    assert _ws(L, chunks=0) == _ws(L, chunks=32)            # 0: the default
    assert _ws(L, lam=-1.0)[0] == INVALID
    assert _ws(L, order=5)[0] == INVALID
    assert _ws(L, topk=9)[0] == INVALID
    assert L.pisa_run_host_workspace(shape(), 2, 1, None, None) == INVALID
    n = ctypes.c_size_t(0)
    assert L.pisa_run_host_workspace(shape(), 2, 1, None, ctypes.byref(n)) == OK   # NULL options: defaults
    assert n.value == _ws(L)[1]
    assert _ws(L, group=9)[0] == INVALID
    assert _ws(L, cand=1)[0] == INVALID             # fewer candidates than topk
    assert _ws(L, group=4, cand=3)[0] == OK


def run_host(L, s=None, topk=2, order=1, scale=0.1, lam=0.0, chunks=2, ws=FAKE, nbytes=None, **ptrs):
    p = {k: FAKE for k in ("Q", "K", "V", "O")}
    p.update(ptrs)
    if nbytes is None:
        nbytes = _ws(L, s, topk, order, lam, chunks)[1]
    return L.pisa_run_host(vp(p["Q"]), vp(p["K"]), vp(p["V"]), s or shape(), topk, order, scale,
                           _opts(lam, chunks), vp(ws), nbytes, vp(p["O"]), None)


def test_host_entry_arguments(L):
    for name in ("Q", "K", "V", "O"):
        assert run_host(L, **{name: 0}) == INVALID, name
    assert run_host(L, ws=0) == INVALID
    assert run_host(L, ws=FAKE + 16) == INVALID          # workspace must be 256-byte aligned
    assert b"256" in L.pisa_last_error()
    assert run_host(L, nbytes=100) == INVALID
    assert b"needed" in L.pisa_last_error()
    assert run_host(L, scale=0.0) == INVALID
    assert run_host(L, chunks=-2) == INVALID
    assert run_host(L, s=shape(B=0), Q=0, K=0, V=0, O=0, ws=0, nbytes=0) == OK
    _no_device()
    _passes_validation(run_host(L, Q=MISALIGNED), L)     # host buffers need no alignment


def test_static_host_entry_arguments(L):
    """pisa_run_host_static: the argument checks of pisa_run_host, and a problem whose
    workspace exceeds the library's fixed region is rejected before any device work."""
    def run(s, topk=2, order=1, chunks=1, **ptrs):
        p = {k: FAKE for k in ("Q", "K", "V", "O")}
        p.update(ptrs)
        return L.pisa_run_host_static(vp(p["Q"]), vp(p["K"]), vp(p["V"]), s, topk, order, 0.1, _opts(0.0, chunks),
                                      vp(p["O"]), None)
    big = shape(B=1, H=2, N=32768, d=128, block=64)              # 64 MiB of Q, K, V, O in one range
    assert _ws(L, big, 64, 1, 0.0, 1)[1] > P.STATIC_WORKSPACE_BYTES
    assert run(big, topk=64) == UNSUPPORTED
    assert b"static region" in L.pisa_last_error()
    assert run(shape(), topk=9) == INVALID                        # topk > nB
    assert run(shape(), order=5) == INVALID
    assert run(shape(B=0), Q=0, K=0, V=0, O=0) == OK               # empty problem: nothing touched
    assert _ws(L, shape(), 2, 1, 0.0, 1)[1] <= P.STATIC_WORKSPACE_BYTES
    for name in ("Q", "K", "V", "O"):
        assert run(shape(), **{name: 0}) == INVALID, name
    _no_device()
    _passes_validation(run(shape()), L)                           # only the device remains


def sel_grouped(L, s=None, Q=FAKE, kbar=FAKE, topk=2, group=2, cand=3, idx=FAKE, route=0, lam=0.0):
    return L.pisa_select_grouped(vp(Q), vp(kbar), vp(route), lam, s or shape(), topk, group, cand, vp(idx), None)


def test_grouped_select_arguments(L):
    assert sel_grouped(L, group=0) == INVALID
    assert sel_grouped(L, group=9) == INVALID
    assert sel_grouped(L, cand=1) == INVALID        # fewer candidates than topk
    assert sel_grouped(L, cand=5) == INVALID        # more candidates than nB = 4
    assert sel_grouped(L, idx=MISALIGNED) == INVALID
    assert sel_grouped(L, s=shape(d=96)) == UNSUPPORTED
    assert sel_grouped(L, s=shape(N=0), Q=0, kbar=0, idx=0) == OK
    _no_device()
    _passes_validation(sel_grouped(L), L)
    _passes_validation(sel_grouped(L, group=8, cand=2), L)

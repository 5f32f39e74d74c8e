"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Small workloads are compared in full; the large video workloads at their full
size on sampled heads and query blocks (the oracle computes those rows one
query block at a time). Tolerances: block indices bit-exact except at rows the
oracle records as near-ties (k-th and (k+1)-th pooled scores within 1e-5
relative); outputs max abs error <= 1e-2 and L1-relative error <= 5e-3.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests import parity as PT

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_sparse_attention_pisa_b200 as P  # noqa: E402


def _skip_without_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.fixture(autouse=True)
def _gpu():
    _skip_without_gpu()
    yield
    P.device_error()          # no kernel may have flagged the device error word


def _inputs(wl, heads=None):
    q, k, v = W.make_inputs(wl, heads)
    dev = [PT.to_device(a) for a in (q, k, v)]
    host = [PT.to_f64(a) for a in (q, k, v)]
    return dev, host


def _check_stats(wl, dq_dk_dv, host, ref=None):
    _, dk, dv = dq_dk_dv
    _, Kf, Vf = host
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, wl.order)
    rk, r0, r1 = oracle.block_stats(Kf, Vf, wl.block, wl.order) if ref is None else ref
    np.testing.assert_allclose(kbar.cpu().numpy(), rk, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(S0.cpu().numpy(), r0, rtol=1e-5, atol=1e-4)
    if wl.order == 1:
        g1 = PT.bf16_to_f64(S1)
        assert np.all(np.abs(g1 - r1) <= 2.0 ** -8 * np.abs(r1) + 1e-3)
    return kbar, S0, S1


SMALL = [
    W.get("tiny"),
    W.get("tiny").with_(order=0),
    W.get("tiny").with_(N=200, topk=3),                       # ragged last block (8 rows)
    W.get("tiny").with_(N=1, topk=1),                         # a single token
    W.get("tiny").with_(d=128, N=330, block=64, topk=2),      # d = 128, ragged
    W.get("tiny").with_(block=128, N=300, topk=1),            # d = 64, b = 128, ragged
    W.get("tiny").with_(d=128, block=128, N=1000, H=3, topk=2, scale=0.09),
    W.get("tiny").with_(N=512, topk=8),                       # all selected: dense attention
    W.get("tiny").with_(N=512, topk=1, H=2, B=2),
    W.get("tiny").with_(d=128, N=330, block=64, topk=2, order=0),   # order 0 at d = 128, b = 64
    W.get("tiny").with_(d=128, N=4096, block=64, topk=5, H=2, order=0),  # two approximate chunks
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: f"{w.name}-N{w.N}-d{w.d}-b{w.block}-k{w.topk}-o{w.order}")
@pytest.mark.parametrize("fn", ["fused", "simt"])
def test_small_pipeline(wl, fn):
    dev, host = _inputs(wl)
    dq, dk, dv = dev
    kbar, S0, S1 = _check_stats(wl, dev, host)
    ref = PT.oracle_pipeline(*host, wl)
    idx = P.select(dq, kbar, wl.block, wl.topk)
    bad, near_bad, _ = PT.compare_idx(idx.cpu().numpy(), ref["idx"], ref["near"],
                                      f"small N{wl.N} d{wl.d} b{wl.block} k{wl.topk} ({fn})")
    assert bad == near_bad, f"{bad} index rows differ, {near_bad} of them at near-ties"
    # the attention is checked on the oracle's own selection
    oidx = torch.from_numpy(ref["idx"]).cuda()
    run = P.attention if fn == "fused" else P.attention_simt
    O = run(dq, dk, dv, kbar, S0, S1, oidx, wl.block, wl.order, wl.scale)
    PT.assert_close(PT.bf16_to_f64(O), ref["O"], f"{fn} {wl}")
    if wl.topk == wl.nB:        # every block exact: equals dense softmax attention
        dense = oracle.dense_attention(*host, wl.scale)
        PT.assert_close(PT.bf16_to_f64(O), dense, "dense equivalence")


def test_clustered_keys_identical_blocks_are_exact():
    """Blocks of identical keys: the order-0 and order-1 outputs equal dense attention."""
    wl = W.get("tiny")
    q, _, v = W.make_inputs(wl)
    k = W.make_clustered_keys(wl, spread=0.0)
    dq, dk, dv = (PT.to_device(a) for a in (q, k, v))
    Qf, Kf, Vf = (PT.to_f64(a) for a in (q, k, v))
    dense = oracle.dense_attention(Qf, Kf, Vf, wl.scale)
    for order in (0, 1):
        kbar, S0, S1 = P.block_stats(dk, dv, wl.block, order)
        idx = P.select(dq, kbar, wl.block, wl.topk)
        O = P.attention(dq, dk, dv, kbar, S0, S1, idx, wl.block, order, wl.scale)
        PT.assert_close(PT.bf16_to_f64(O), dense, f"identical keys, order {order}")


def test_clustered_keys_order1_beats_order0():
    wl = W.get("tiny")
    q, _, v = W.make_inputs(wl)
    k = W.make_clustered_keys(wl, spread=0.1)
    dq, dk, dv = (PT.to_device(a) for a in (q, k, v))
    Qf, Kf, Vf = (PT.to_f64(a) for a in (q, k, v))
    dense = oracle.dense_attention(Qf, Kf, Vf, wl.scale)
    errs = {}
    for order in (0, 1):
        ref = PT.oracle_pipeline(Qf, Kf, Vf, wl.with_(order=order))
        kbar, S0, S1 = P.block_stats(dk, dv, wl.block, order)
        oidx = torch.from_numpy(ref["idx"]).cuda()
        O = P.attention(dq, dk, dv, kbar, S0, S1, oidx, wl.block, order, wl.scale)
        PT.assert_close(PT.bf16_to_f64(O), ref["O"], f"clustered order {order}")
        errs[order] = np.abs(PT.bf16_to_f64(O) - dense).mean()
    assert errs[1] < errs[0]


@pytest.mark.parametrize("name", ["image", "dense", "dense_k8_o0", "dense_k8_o1"])
def test_full_workload(name):
    wl = W.get(name)
    dev, host = _inputs(wl)
    dq, dk, dv = dev
    kbar, S0, S1 = _check_stats(wl, dev, host)
    ref = PT.oracle_pipeline(*host, wl)
    idx = P.select(dq, kbar, wl.block, wl.topk)
    bad, near_bad, bad_rows = PT.compare_idx(idx.cpu().numpy(), ref["idx"], ref["near"], name)
    assert bad == near_bad, f"{bad} index rows differ, {near_bad} at near-ties"
    O = P.attention(dq, dk, dv, kbar, S0, S1, idx, wl.block, wl.order, wl.scale)
    out = PT.bf16_to_f64(O)
    # rows of query blocks whose selection differs at a near-tie are not comparable
    mask = np.repeat(~bad_rows, wl.block, axis=-1)[..., :wl.N, None]
    PT.assert_close(np.where(mask, out, 0.0), np.where(mask, ref["O"], 0.0), name)
    if wl.topk == wl.nB:
        dense = oracle.dense_attention(*host, wl.scale)
        PT.assert_close(out, dense, "dense equivalence")


@pytest.mark.parametrize("name", ["video", "long"])
def test_large_workload_sampled(name):
    """Full-size launch; the oracle checks three heads on 32 sampled query blocks each
    (at b = 64 both query blocks of 16 of the 128-row tiles, first and last included)."""
    wl = W.get(name)
    q, k, v = W.make_inputs(wl)
    dq, dk, dv = (PT.to_device(a) for a in (q, k, v))
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, wl.order)
    idx = P.select(dq, kbar, wl.block, wl.topk)
    O = P.attention(dq, dk, dv, kbar, S0, S1, idx, wl.block, wl.order, wl.scale)
    torch.cuda.synchronize()
    heads = [0, wl.H // 2, wl.H - 1]
    qbs = PT.sampled_query_blocks(wl, 32)
    sub = wl.with_(H=len(heads))
    Qf, Kf, Vf = (PT.to_f64(a[:, heads]) for a in (q, k, v))
    rk, r0, r1 = oracle.block_stats(Kf, Vf, wl.block, wl.order)
    np.testing.assert_allclose(kbar[:, heads].cpu().numpy(), rk, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(S0[:, heads].cpu().numpy(), r0, rtol=1e-5, atol=1e-4)
    g1 = PT.bf16_to_f64(S1[:, heads])
    assert np.all(np.abs(g1 - r1) <= 2.0 ** -8 * np.abs(r1) + 1e-3)
    ridx, near, _ = oracle.select(Qf, rk, wl.block, wl.topk)
    gidx = idx[:, heads].cpu().numpy()
    bad, near_bad, bad_rows = PT.compare_idx(gidx, ridx, near, f"{name} (3 heads)")
    assert bad == near_bad, f"{bad} index rows differ, {near_bad} at near-ties"
    ref = oracle.attention(Qf, Kf, Vf, rk, r0, r1, ridx, wl.block, wl.order, wl.scale,
                           query_blocks=qbs)
    out = PT.bf16_to_f64(O[:, heads])
    rows = np.concatenate([np.arange(i * wl.block, min((i + 1) * wl.block, wl.N)) for i in qbs
                           if not bad_rows[0, :, i].any()])
    PT.assert_close(out[:, :, rows], ref[:, :, rows], f"{name} sampled")
    del sub


def test_deterministic():
    wl = W.get("image").with_(B=1, H=4)
    (dq, dk, dv), _ = _inputs(wl)
    outs = []
    for _ in range(2):
        O, idx = P.pisa(dq, dk, dv, wl.block, wl.topk, wl.order, wl.scale)
        outs.append((O.clone(), idx.clone()))
    assert torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16))


def test_out_of_range_index_is_flagged_not_faulted():
    """An idx entry outside [0, nB) is skipped by the kernel's bounds check and reported."""
    wl = W.get("tiny")
    (dq, dk, dv), _ = _inputs(wl)
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, wl.order)
    idx = P.select(dq, kbar, wl.block, wl.topk)
    idx[0, 0, 1, 0] = wl.nB + 5
    for run in (P.attention, P.attention_simt):
        run(dq, dk, dv, kbar, S0, S1, idx, wl.block, wl.order, wl.scale)
        with pytest.raises(P.PisaError, match="INVALID_ARG"):
            P.device_error()


def test_device_error_word_is_shared_per_device():
    """A bit raised by a kernel on one stream is reported by a device_error call on another
    stream (the word is one per device), and that call clears it."""
    wl = W.get("tiny")
    (dq, dk, dv), _ = _inputs(wl)
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, wl.order)
    idx = P.select(dq, kbar, wl.block, wl.topk)
    idx[0, 0, 2, 1] = -3
    P.attention(dq, dk, dv, kbar, S0, S1, idx, wl.block, wl.order, wl.scale)
    torch.cuda.synchronize()
    other = torch.cuda.Stream()
    with torch.cuda.stream(other):
        with pytest.raises(P.PisaError, match="INVALID_ARG"):
            P.device_error()
    P.device_error()          # taken by the first reader: nothing left


@pytest.mark.parametrize("order,lam,group,cand", [(1, 0.0, 1, 0), (2, 0.0, 1, 0), (-1, 0.0, 1, 0), (0, 0.0, 1, 0),
                                                  (2, 0.02, 1, 0), (1, 0.02, 1, 0), (2, 0.0, 4, 32), (1, 0.02, 2, 16)])
def test_host_entry_point_matches_device(order, lam, group, cand):
    """pisa_run_host (host buffers in and out, through the C ABI) gives the bits of the
    device calls on the whole batch, for every order, with and without routing and with
    grouped selection."""
    wl = W.get("image").with_(B=1, H=2)
    q, k, v = W.make_inputs(wl)
    hq, hk, hv = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in (q, k, v))
    Oh = P.pisa_host(hq, hk, hv, wl.block, wl.topk, order, wl.scale, route_lambda=lam, group=group, candidates=cand)
    Od, _ = P.pisa(hq.cuda(), hk.cuda(), hv.cuda(), wl.block, wl.topk, order, wl.scale, route_lambda=lam,
                   group=group, candidates=cand or None)
    assert torch.equal(Oh.view(torch.int16), Od.cpu().view(torch.int16))


def test_host_entry_point_pipelined_over_heads():
    """The host entry point splits (batch, head) pairs into ranges that copy and compute
    on separate streams through three workspace slots; every chunking gives the device
    path's bits, with page-locked and with pageable host memory."""
    wl = W.get("image").with_(B=2, H=3)
    q, k, v = W.make_inputs(wl)
    hq, hk, hv = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in (q, k, v))
    Od, _ = P.pisa(hq.cuda(), hk.cuda(), hv.cuda(), wl.block, wl.topk, wl.order, wl.scale)
    ref = Od.cpu().view(torch.int16)
    for chunks in (1, 2, 4, 6, 16):
        Oh = P.pisa_host(hq, hk, hv, wl.block, wl.topk, wl.order, wl.scale, chunks=chunks)
        assert torch.equal(Oh.view(torch.int16), ref), chunks
    pq, pk, pv = (t.clone() for t in (hq, hk, hv))       # pageable copies
    assert not pq.is_pinned()
    Oh = P.pisa_host(pq, pk, pv, wl.block, wl.topk, wl.order, wl.scale, chunks=4)
    assert torch.equal(Oh.view(torch.int16), ref)


def test_host_entry_point_rejects_device_buffers():
    wl = W.get("tiny")
    q, k, v = (PT.to_device(a) for a in W.make_inputs(wl))
    s = P.Shape(wl.B, wl.H, wl.N, wl.d, wl.block)
    n = P.host_workspace_bytes(s, wl.topk, wl.order)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    O = torch.empty_like(q)
    st = P.lib().pisa_run_host(P._ptr(q), P._ptr(k), P._ptr(v), s, wl.topk, wl.order, wl.scale, None,
                               P._ptr(ws), n, P._ptr(O), None)
    assert st == 1 and b"device memory" in P.lib().pisa_last_error()

"""Keep-or-drop (order -1) and the hybrid order with the global Hbar (order 2):
the CUDA path vs the CPU oracle through the C ABI.

Same tolerances as the other parity tests (outputs max abs error <= 1e-2 and
L1-relative error <= 5e-3; block indices bit-exact except at recorded
near-ties). Hbar is an fp32 sum of fp32 terms: within 1e-4 of its largest entry.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests import parity as PT

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_sparse_attention_pisa_b200 as P  # noqa: E402


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    P.device_error()          # no kernel may have flagged the device error word


def _inputs(wl, heads=None):
    q, k, v = W.make_inputs(wl, heads)
    return [PT.to_device(a) for a in (q, k, v)], [PT.to_f64(a) for a in (q, k, v)]


SMALL = [
    W.get("tiny"),
    W.get("tiny").with_(N=200, topk=3),                       # ragged last block (8 rows)
    W.get("tiny").with_(N=1, topk=1),                         # a single token
    W.get("tiny").with_(d=128, N=330, block=64, topk=2),      # d = 128, ragged
    W.get("tiny").with_(block=128, N=300, topk=1),            # d = 64, b = 128, ragged
    W.get("tiny").with_(d=128, block=128, N=1000, H=3, topk=2, scale=0.09),
    W.get("tiny").with_(N=512, topk=8),                       # all selected: dense attention
    W.get("tiny").with_(N=4096, topk=5, H=2, B=2),            # 64 blocks: two approximate chunks
]


@pytest.mark.parametrize("order", [-1, 2])
@pytest.mark.parametrize("wl", SMALL, ids=lambda w: f"N{w.N}-d{w.d}-b{w.block}-k{w.topk}")
@pytest.mark.parametrize("fn", ["fused", "simt"])
def test_small_pipeline(wl, order, fn):
    wl = wl.with_(order=order)
    (dq, dk, dv), host = _inputs(wl)
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, order)
    ref = PT.oracle_pipeline(*host, wl)
    np.testing.assert_allclose(kbar.cpu().numpy(), ref["kbar"], rtol=1e-5, atol=1e-5)
    PT.check_first_order_stat(S1, ref["S1"], order)
    idx = P.select(dq, kbar, wl.block, wl.topk)
    bad, near_bad, _ = PT.compare_idx(idx.cpu().numpy(), ref["idx"], ref["near"],
                                      f"order {order} N{wl.N} d{wl.d} b{wl.block} ({fn})")
    assert bad == near_bad, f"{bad} index rows differ, {near_bad} of them at near-ties"
    oidx = torch.from_numpy(ref["idx"]).cuda()
    run = P.attention if fn == "fused" else P.attention_simt
    if order == -1:             # keep-or-drop reads no block statistics
        O = run(dq, dk, dv, None, None, None, oidx, wl.block, order, wl.scale)
    else:
        O = run(dq, dk, dv, kbar, S0, S1, oidx, wl.block, order, wl.scale)
    PT.assert_close(PT.bf16_to_f64(O), ref["O"], f"{fn} order {order} {wl}")
    if wl.topk == wl.nB:
        PT.assert_close(PT.bf16_to_f64(O), oracle.dense_attention(*host, wl.scale), "dense equivalence")


def test_hybrid_equals_first_order_for_shared_pattern():
    """Blocks that are translated copies of one key/value pattern share one first-order
    matrix, so on the GPU too the hybrid output matches the per-block first order."""
    wl = W.get("tiny").with_(d=128, N=2048, topk=3)
    rng = np.random.default_rng(7)
    c = rng.standard_normal((wl.nB, wl.d)).astype(np.float32)
    z = 0.3 * rng.standard_normal((wl.block, wl.d)).astype(np.float32)
    u = rng.standard_normal((wl.block, wl.d)).astype(np.float32)
    k = W.to_bf16_bits((np.repeat(c, wl.block, axis=0) + np.tile(z, (wl.nB, 1)))[None, None])
    v = W.to_bf16_bits(np.tile(u, (wl.nB, 1))[None, None])
    q = W.make_inputs(wl)[0]
    dq, dk, dv = (PT.to_device(a) for a in (q, k, v))
    outs = {}
    for order in (1, 2):
        kbar, S0, S1 = P.block_stats(dk, dv, wl.block, order)
        idx = P.select(dq, kbar, wl.block, wl.topk)
        outs[order] = PT.bf16_to_f64(P.attention(dq, dk, dv, kbar, S0, S1, idx, wl.block, order, wl.scale))
    PT.assert_close(outs[2], outs[1], "hybrid vs first order, shared pattern")


@pytest.mark.parametrize("order", [-1, 2])
def test_image_workload(order):
    wl = W.get("image").with_(order=order)
    (dq, dk, dv), host = _inputs(wl)
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, order)
    ref = PT.oracle_pipeline(*host, wl)
    PT.check_first_order_stat(S1, ref["S1"], order)
    idx = P.select(dq, kbar, wl.block, wl.topk)
    bad, near_bad, bad_rows = PT.compare_idx(idx.cpu().numpy(), ref["idx"], ref["near"], f"image order {order}")
    assert bad == near_bad
    O = P.attention(dq, dk, dv, kbar, S0, S1, idx, wl.block, order, wl.scale)
    out = PT.bf16_to_f64(O)
    mask = np.repeat(~bad_rows, wl.block, axis=-1)[..., :wl.N, None]
    PT.assert_close(np.where(mask, out, 0.0), np.where(mask, ref["O"], 0.0), f"image order {order}")


@pytest.mark.parametrize("name", ["video_hybrid", "video_drop", "long_hybrid"])
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
    Qf, Kf, Vf = (PT.to_f64(a[:, heads]) for a in (q, k, v))
    rk, r0, r1 = PT.oracle_stats(Kf, Vf, wl)
    np.testing.assert_allclose(kbar[:, heads].cpu().numpy(), rk, rtol=1e-5, atol=1e-5)
    if wl.order == 2:
        PT.check_first_order_stat(S1[:, heads], r1, 2)
    ridx, near, _ = oracle.select(Qf, rk, wl.block, wl.topk)
    bad, near_bad, bad_rows = PT.compare_idx(idx[:, heads].cpu().numpy(), ridx, near, f"{name} (3 heads)")
    assert bad == near_bad, f"{bad} index rows differ, {near_bad} at near-ties"
    ref = oracle.attention(Qf, Kf, Vf, rk, r0, r1, ridx, wl.block, wl.order, wl.scale,
                           query_blocks=qbs)
    out = PT.bf16_to_f64(O[:, heads])
    rows = np.concatenate([np.arange(i * wl.block, min((i + 1) * wl.block, wl.N)) for i in qbs
                           if not bad_rows[0, :, i].any()])
    PT.assert_close(out[:, :, rows], ref[:, :, rows], f"{name} sampled")


def test_drop_deterministic():
    wl = W.get("image").with_(B=1, H=4, order=-1)
    (dq, dk, dv), _ = _inputs(wl)
    a, ia = P.pisa(dq, dk, dv, wl.block, wl.topk, -1, wl.scale)
    b, ib = P.pisa(dq, dk, dv, wl.block, wl.topk, -1, wl.scale)
    assert torch.equal(ia, ib) and torch.equal(a.view(torch.int16), b.view(torch.int16))

"""Covariance-aware routing on the GPU vs the CPU oracle, through the C ABI.

The routing statistic (Hbar and M_j = ||S1_j - Hbar||_F from the stored bf16
S1) is an fp32 sum of fp32 terms: within 1e-4 relative. Block indices are
bit-exact except at rows the oracle records as near-ties; outputs meet the
usual 1e-2 max abs / 5e-3 L1-relative tolerance.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests import parity as PT

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_sparse_attention_pisa_b200 as P  # noqa: E402

LAM = 0.02


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    P.device_error()


def _inputs(wl, heads=None):
    q, k, v = W.make_inputs(wl, heads)
    return [PT.to_device(a) for a in (q, k, v)], [PT.to_f64(a) for a in (q, k, v)]


def _check_routing(Hbar, M, S1_ref, S1_gpu):
    """M and Hbar against the oracle. The GPU's stored S1 may sit one bf16 step away
    from the oracle's rounding of its fp64 S1 where the fp32 value lies on a rounding
    boundary, so Hbar is also checked exactly against the mean of the GPU's own S1."""
    ref_M = oracle.routing_norms(S1_ref)
    ref_H = oracle.round_to_bf16(S1_ref).mean(axis=2)
    nB = S1_ref.shape[2]
    g_M = M.double().cpu().numpy()
    g_H = Hbar.double().cpu().numpy()
    assert np.abs(g_M - ref_M).max() <= 1e-4 * np.abs(ref_M).max(), np.abs(g_M - ref_M).max()
    own_H = PT.bf16_to_f64(S1_gpu).mean(axis=2)
    assert np.abs(g_H - own_H).max() <= 1e-5 * np.abs(own_H).max() + 1e-6
    ulp = 2.0 ** -7 * np.abs(S1_ref).max()        # one bf16 step at the largest entry
    assert np.abs(g_H - ref_H).max() <= 4 * ulp / nB
    return ref_M, ref_H


SMALL = [
    W.get("tiny"),
    W.get("tiny").with_(N=200, topk=3),                       # ragged last block
    W.get("tiny").with_(d=128, N=330, block=64, topk=2),
    W.get("tiny").with_(block=128, N=300, topk=1),
    W.get("tiny").with_(d=128, block=128, N=1000, H=3, topk=2, scale=0.09),
    W.get("tiny").with_(N=4096, topk=5, H=2, B=2),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: f"N{w.N}-d{w.d}-b{w.block}-k{w.topk}")
def test_routed_hybrid_pipeline(wl):
    """stats (order 1) -> routing norms -> routed select -> hybrid attention with that Hbar."""
    (dq, dk, dv), (Qf, Kf, Vf) = _inputs(wl)
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, 1)
    Hbar, M = P.routing_norms(S1, wl.block, wl.N)
    rk, r0, r1 = oracle.block_stats(Kf, Vf, wl.block, 1)
    ref_M, ref_H = _check_routing(Hbar, M, r1, S1)
    idx = P.select(dq, kbar, wl.block, wl.topk, route=M, lam=LAM)
    ridx, near, _ = oracle.select(Qf, rk, wl.block, wl.topk, route=ref_M, lam=LAM)
    bad, near_bad, _ = PT.compare_idx(idx.cpu().numpy(), ridx, near, f"routed N{wl.N} d{wl.d} b{wl.block}")
    assert bad == near_bad, f"{bad} index rows differ, {near_bad} of them at near-ties"
    O = P.attention(dq, dk, dv, kbar, S0, Hbar, torch.from_numpy(ridx).cuda(), wl.block, 2, wl.scale)
    ref = oracle.attention(Qf, Kf, Vf, rk, r0, ref_H, ridx, wl.block, 2, wl.scale)
    PT.assert_close(PT.bf16_to_f64(O), ref, f"routed hybrid {wl}")


def test_zero_weight_is_plain_relevance():
    wl = W.get("image").with_(B=1, H=4)
    (dq, dk, dv), _ = _inputs(wl)
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, 1)
    _, M = P.routing_norms(S1, wl.block, wl.N)
    assert torch.equal(P.select(dq, kbar, wl.block, wl.topk, route=M, lam=0.0),
                       P.select(dq, kbar, wl.block, wl.topk))


@pytest.mark.parametrize("name", ["image", "video_routed"])
def test_routing_full_size(name):
    """Full-size launch: routing statistic and routed indices on sampled heads; the
    weight changes the selection of a fair share of rows."""
    wl = W.get(name)
    lam = wl.route_lambda or LAM
    q, k, v = W.make_inputs(wl)
    dq, dk, dv = (PT.to_device(a) for a in (q, k, v))
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, 1)
    Hbar, M = P.routing_norms(S1, wl.block, wl.N)
    idx = P.select(dq, kbar, wl.block, wl.topk, route=M, lam=lam)
    plain = P.select(dq, kbar, wl.block, wl.topk)
    torch.cuda.synchronize()
    changed = (idx != plain).any(-1).float().mean().item()
    assert changed > 0.05, f"routing changed only {changed:.3f} of the rows"
    heads = [0, wl.H - 1]
    bi = 0
    Qf, Kf, Vf = (PT.to_f64(a[bi:bi + 1, heads]) for a in (q, k, v))
    rk, r0, r1 = oracle.block_stats(Kf, Vf, wl.block, 1)
    sub = lambda t: t[bi:bi + 1, heads]  # noqa: E731
    ref_M, ref_H = _check_routing(sub(Hbar), sub(M), r1, sub(S1))
    ridx, near, _ = oracle.select(Qf, rk, wl.block, wl.topk, route=ref_M, lam=lam)
    bad, near_bad, _ = PT.compare_idx(sub(idx).cpu().numpy(), ridx, near, f"{name} routed (2 heads)")
    assert bad == near_bad, f"{bad} index rows differ, {near_bad} at near-ties"

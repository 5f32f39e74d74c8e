"""Grouped-proxy selection (selection amortisation) on the GPU against the oracle.

PIVOT page, "Two observations behind PIVOT": one proxy query per group of query blocks
(the mean of the group's real rows) keeps a candidate list, and every member keeps its
own best topk of those candidates; candidates = topk is the reuse mode. Block indices
must equal the oracle's (``oracle.select_grouped``) bit for bit, except at rows the
oracle flags as near-ties (at the proxy's or the member's cut, 1e-5 relative).
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
    P.device_error()


CASES = [  # (workload, group, candidates)
    (W.get("tiny").with_(N=1024, topk=3), 2, 3),                         # reuse
    (W.get("tiny").with_(N=1024, topk=3), 4, 6),                         # refine
    (W.get("tiny").with_(N=1000, topk=2, H=2), 3, 5),                    # ragged, group of 3
    (W.get("tiny").with_(d=128, N=4096 - 17, topk=8), 8, 16),            # d = 128, ragged
    (W.get("tiny").with_(d=128, N=128 * 40 - 9, block=128, topk=4), 4, 9),  # b = 128
    (W.get("tiny").with_(d=64, N=64 * 70, topk=5, B=2), 5, 12),          # a group of 5, tile of 5
    (W.get("tiny").with_(N=1024, topk=3), 1, 7),                         # own proxy: plain selection
    (W.get("tiny").with_(N=2048, topk=4), 6, 32),                        # all candidates: plain
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"N{c[0].N}-d{c[0].d}-b{c[0].block}-k{c[0].topk}-g{c[1]}-c{c[2]}")
@pytest.mark.parametrize("routed", [False, True])
def test_grouped_select_matches_oracle(case, routed):
    wl, g, c = case
    q, k, v = W.make_inputs(wl)
    dq, dk, dv = (PT.to_device(a) for a in (q, k, v))
    Qf, Kf, Vf = (PT.to_f64(a) for a in (q, k, v))
    kbar, _, S1 = P.block_stats(dk, dv, wl.block, 1 if routed else 0)
    rk, _, r1 = oracle.block_stats(Kf, Vf, wl.block, 1 if routed else 0)
    lam = 0.02 if routed else 0.0
    M = ref_M = None
    if routed:
        _, M = P.routing_norms(S1, wl.block, wl.N)
        ref_M = oracle.routing_norms(r1)
    idx = P.select(dq, kbar, wl.block, wl.topk, route=M, lam=lam, group=g, candidates=c)
    ridx, near = oracle.select_grouped(Qf, rk, wl.block, wl.topk, g, c, route=ref_M, lam=lam)
    bad, near_bad, _ = PT.compare_idx(idx.cpu().numpy(), ridx, near, f"grouped g{g} c{c} N{wl.N} d{wl.d}")
    assert bad == near_bad, f"{bad} index rows differ, {near_bad} of them at near-ties"
    if c == wl.topk:                 # reuse: members of a group share their row
        got = idx.cpu().numpy()
        for m in range(-(-wl.nB // g)):
            rows = got[:, :, m * g:(m + 1) * g]
            assert (rows == rows[:, :, :1]).all()


@pytest.mark.parametrize("g,c", [(4, 128), (8, 64)])
def test_grouped_video_workload(g, c):
    """Full-size video launch: grouped indices on three heads against the oracle, then
    the attention computed on them against the oracle on sampled query blocks."""
    wl = W.get("video")
    q, k, v = W.make_inputs(wl)
    dq, dk, dv = (PT.to_device(a) for a in (q, k, v))
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, wl.order)
    idx = P.select(dq, kbar, wl.block, wl.topk, group=g, candidates=c)
    O = P.attention(dq, dk, dv, kbar, S0, S1, idx, wl.block, wl.order, wl.scale)
    torch.cuda.synchronize()
    heads = [0, wl.H // 2, wl.H - 1]
    Qf, Kf, Vf = (PT.to_f64(a[:, heads]) for a in (q, k, v))
    rk, r0, r1 = oracle.block_stats(Kf, Vf, wl.block, wl.order)
    ridx, near = oracle.select_grouped(Qf, rk, wl.block, wl.topk, g, c)
    bad, near_bad, bad_rows = PT.compare_idx(idx[:, heads].cpu().numpy(), ridx, near, f"video grouped g{g} c{c}")
    assert bad == near_bad, f"{bad} index rows differ, {near_bad} at near-ties"
    qbs = PT.sampled_query_blocks(wl, 16)
    ref = oracle.attention(Qf, Kf, Vf, rk, r0, r1, ridx, wl.block, wl.order, wl.scale, query_blocks=qbs)
    rows = np.concatenate([np.arange(i * wl.block, (i + 1) * wl.block) for i in qbs if not bad_rows[0, :, i].any()])
    PT.assert_close(PT.bf16_to_f64(O[:, heads])[:, :, rows], ref[:, :, rows], f"video grouped g{g} c{c}")

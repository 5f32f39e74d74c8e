"""Running-maximum rescales of the fused kernel, forced on purpose, against the oracle.

The fused kernel keeps one running row maximum over the exact and the approximate
stage and rescales the accumulator (numerator and denominator) only when the maximum
grows by more than 2^8 in base-2 units. Inputs with logits of unit spread never grow
it that much after the first block, so these cases plant "hot" key blocks whose
logits sit 12-25 natural-log units above everything seen before them:

* exact stage: the hot blocks are selected and visited after ordinary ones;
* approximate stage: a hot block is left out of a query block's selection, so its
  pooled score exp(x . kbar) jumps above every exact score, in the first or a later
  chunk of 32 approximated blocks, and for one or both query blocks of a 128-row tile.

All exponents stay relative to one maximum in the explainer's o_t = N_t / D_t (section 2,
"Core algorithm"), so the rescaled output must match the oracle like any other.
Tolerances as everywhere: max abs error <= 1e-2, L1-relative error <= 5e-3.
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


def _hot_inputs(wl, hot, lift=3.0):
    """Q, K, V (bf16 bits) with every query lifted by `lift` along dimension 0 and each
    key of block j in `hot` lifted by hot[j] along the same dimension: the logits of that
    block rise by about scale * lift * hot[j] for every query."""
    q, k, v = W.make_inputs(wl)
    Qf, Kf = (W.bf16_bits_to_f32(a).copy() for a in (q, k))
    Qf[..., 0] += lift
    for j, c in hot.items():
        Kf[:, :, j * wl.block:min((j + 1) * wl.block, wl.N), 0] += c
    return W.to_bf16_bits(Qf), W.to_bf16_bits(Kf), v


def _lift_for(wl, natural, lift=3.0):
    """Key lift that raises a block's logits by about `natural` (natural-log units)."""
    return natural / (wl.scale * lift)


def _run(wl, q, k, v, idx, order, fns=("fused", "simt")):
    dq, dk, dv = (PT.to_device(a) for a in (q, k, v))
    Qf, Kf, Vf = (PT.to_f64(a) for a in (q, k, v))
    kbar, S0, S1 = P.block_stats(dk, dv, wl.block, order)
    rk, r0, r1 = PT.oracle_stats(Kf, Vf, wl.with_(order=order))
    ref = oracle.attention(Qf, Kf, Vf, rk, r0, r1, idx, wl.block, order, wl.scale)
    didx = torch.from_numpy(idx).cuda()
    for fn in fns:
        run = P.attention if fn == "fused" else P.attention_simt
        O = run(dq, dk, dv, kbar, S0, S1, didx, wl.block, order, wl.scale)
        PT.assert_close(PT.bf16_to_f64(O), ref, f"{fn} order {order}")
    return ref


EXACT_CASES = [
    W.get("tiny").with_(d=128, N=1024, block=64, topk=4),           # d = 128, b = 64
    W.get("tiny").with_(d=64, N=1000, block=64, topk=4),            # d = 64, ragged
    W.get("tiny").with_(d=128, N=2048 - 40, block=128, topk=4),     # b = 128, ragged
]


@pytest.mark.parametrize("order", [-1, 0, 1, 2])
@pytest.mark.parametrize("wl", EXACT_CASES, ids=lambda w: f"d{w.d}-b{w.block}-N{w.N}")
def test_exact_stage_rescale(wl, order):
    """Selected blocks [0, 1, 2, mid, last]: `mid` sits ~12 above blocks 0-2 and `last`
    ~25 above them, so the maximum grows twice after the first blocks' P V are issued."""
    mid, last = wl.nB // 2, wl.nB - 1
    hot = {mid: _lift_for(wl, 12.0), last: _lift_for(wl, 25.0)}
    q, k, v = _hot_inputs(wl, hot)
    sel = np.array(sorted({0, 1, 2, mid, last}), dtype=np.int32)
    idx = np.broadcast_to(sel, (wl.B, wl.H, wl.nB, sel.size)).copy()
    ref = _run(wl, q, k, v, idx, order)
    assert np.isfinite(ref).all()


APPROX_CASES = [
    (W.get("tiny").with_(d=128, N=4096, block=64, topk=5), 50),     # hot block in chunk 1 of 2
    (W.get("tiny").with_(d=128, N=4096, block=64, topk=5), 7),      # hot block in chunk 0
    (W.get("tiny").with_(d=64, N=64 * 70 - 9, block=64, topk=3), 66),  # chunk 2 of 3, ragged
    (W.get("tiny").with_(d=128, N=128 * 40, block=128, topk=4), 33),    # b = 128, chunk 1
]


@pytest.mark.parametrize("order", [0, 1, 2])
@pytest.mark.parametrize("case", APPROX_CASES, ids=lambda c: f"d{c[0].d}-b{c[0].block}-N{c[0].N}-hot{c[1]}")
def test_approximate_stage_rescale(case, order):
    """One key block, ~15 above every exact score, is selected by the even query blocks and
    approximated by the odd ones: in each 128-row tile at b = 64 one query block treats it
    exactly and the other meets it first as a pooled score in the approximate stage."""
    wl, hot_j = case
    q, k, v = _hot_inputs(wl, {hot_j: _lift_for(wl, 15.0)})
    rng = np.random.default_rng(5)
    idx = np.empty((wl.B, wl.H, wl.nB, wl.topk), dtype=np.int32)
    others = np.array([j for j in range(wl.nB) if j != hot_j])
    for b in range(wl.B):
        for h in range(wl.H):
            for i in range(wl.nB):
                pick = rng.choice(others, size=wl.topk, replace=False)
                if i % 2 == 0:
                    pick[0] = hot_j
                idx[b, h, i] = np.sort(pick)
    _run(wl, q, k, v, idx, order)

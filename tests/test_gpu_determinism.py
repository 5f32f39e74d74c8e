"""The hybrid order's statistics are the same bits on every call (GPU).

PISA explainer, technical summary section 2, "Core algorithm": the hybrid order's Hbar is
the mean of the per-block first-order matrices over a head's blocks; "Covariance-aware
routing": M_j = ||S1_j - Hbar||_F. The kernels split each head's blocks into a fixed
number of contiguous slices and add the partial sums in a fixed order, without atomics.
So Hbar and M, and with them the hybrid order's output, repeat bit for bit. A head's
statistics also do not depend on which other heads share the launch. Block counts
below the slice count leave some slices empty; keys with a large common mean make
the per-slice sums cancel, and Hbar must still meet the oracle's tolerance.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_pisa_b200 as P
import oracle
from tests import parity as PT
import workloads as W

pytestmark = pytest.mark.gpu

# (d, block, N): several slices per head, ragged tails, and nB = 2, 3 (< 4 slices)
CASES = [(128, 64, 4096), (128, 128, 4000), (64, 64, 4096), (64, 128, 3000),
         (128, 64, 100), (64, 64, 130), (128, 128, 300)]


def _bits_equal(a, b):
    return torch.equal(a.contiguous().view(torch.int32), b.contiguous().view(torch.int32))


def _wl(d, block, N, order):
    return W.get("tiny").with_(B=2, H=3, N=N, d=d, block=block, order=order, topk=1, scale=d ** -0.5)


@pytest.mark.parametrize("d,block,N", CASES)
def test_hbar_repeats_and_is_per_head(d, block, N):
    wl = _wl(d, block, N, 2)
    q, k, v = W.make_inputs(wl)
    dk, dv = PT.to_device(k), PT.to_device(v)
    kb, s0, hb = P.block_stats(dk, dv, block, 2)
    _, _, hb2 = P.block_stats(dk, dv, block, 2)
    torch.cuda.synchronize()
    P.device_error()
    assert _bits_equal(hb, hb2)
    for b in range(wl.B):
        for h in range(wl.H):
            kb1, s01, hb1 = P.block_stats(dk[b:b + 1, h:h + 1].contiguous(), dv[b:b + 1, h:h + 1].contiguous(), block, 2)
            assert _bits_equal(hb1[0, 0], hb[b, h]), (b, h)
            assert _bits_equal(kb1[0, 0], kb[b, h]) and _bits_equal(s01[0, 0], s0[b, h]), (b, h)
    _, _, r1 = PT.oracle_stats(PT.to_f64(k), PT.to_f64(v), wl)
    PT.check_first_order_stat(hb, r1, 2)


@pytest.mark.parametrize("d,block", [(128, 64), (64, 128)])
def test_hbar_with_a_large_key_mean(d, block):
    wl = _wl(d, block, 8192, 2)
    q, k, v = W.make_inputs(wl)
    kf = W.bf16_bits_to_f32(k) + 4.0            # keys centred at 4: the slice sums cancel
    k = W.to_bf16_bits(kf)
    _, _, hb = P.block_stats(PT.to_device(k), PT.to_device(v), block, 2)
    torch.cuda.synchronize()
    _, _, r1 = PT.oracle_stats(PT.to_f64(k), PT.to_f64(v), wl)
    PT.check_first_order_stat(hb, r1, 2)


@pytest.mark.parametrize("d,block,N", [(128, 64, 4096), (64, 128, 3000), (128, 128, 300)])
def test_routing_norms_repeat_and_are_per_head(d, block, N):
    wl = _wl(d, block, N, 1)
    q, k, v = W.make_inputs(wl)
    dk, dv = PT.to_device(k), PT.to_device(v)
    _, _, S1 = P.block_stats(dk, dv, block, 1)
    H1, M1 = P.routing_norms(S1, block, N)
    H2, M2 = P.routing_norms(S1, block, N)
    torch.cuda.synchronize()
    P.device_error()
    assert _bits_equal(H1, H2) and _bits_equal(M1, M2)
    Hs, Ms = P.routing_norms(S1[1:2, 2:3].contiguous(), block, N)
    assert _bits_equal(Hs[0, 0], H1[1, 2]) and _bits_equal(Ms[0, 0], M1[1, 2])
    # against the oracle on the stored (bf16) S1
    S1f = S1.double().cpu().numpy()
    Hbar = oracle.global_first_order(S1f)
    np.testing.assert_allclose(H1.double().cpu().numpy(), Hbar, rtol=0, atol=1e-5 * np.abs(Hbar).max() + 1e-7)
    M = oracle.routing_norms(S1f)            # S1f holds the stored bf16 values already
    np.testing.assert_allclose(M1.double().cpu().numpy(), M, rtol=1e-4, atol=1e-6)


@pytest.mark.parametrize("route_lambda", [0.0, 0.02])
def test_hybrid_output_repeats(route_lambda):
    wl = W.get("image").with_(B=1, H=3, order=2)
    q, k, v = W.make_inputs(wl)
    dq, dk, dv = PT.to_device(q), PT.to_device(k), PT.to_device(v)
    a, ia = P.pisa(dq, dk, dv, wl.block, wl.topk, 2, wl.scale, route_lambda=route_lambda)
    b, ib = P.pisa(dq, dk, dv, wl.block, wl.topk, 2, wl.scale, route_lambda=route_lambda)
    torch.cuda.synchronize()
    P.device_error()
    assert torch.equal(ia, ib)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))

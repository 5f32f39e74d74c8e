"""The entry point that allocates nothing, ``pisa_run_host_static`` (GPU).

Its device workspace is the library's own fixed region (32 MiB per device); otherwise it
is ``pisa_run_host``. Two calls in a row must each give the bits that the
caller-workspace entry point gives on the same inputs, at every order. The file is
collected last, after every other test has run on the same device.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_pisa_b200 as P
import workloads as W

pytestmark = pytest.mark.gpu


def _host_inputs(wl):
    q, k, v = W.make_inputs(wl)
    return tuple(torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in (q, k, v))


@pytest.mark.parametrize("order,chunks", [(1, 2), (-1, 8), (2, 3)])
def test_static_workspace_matches_caller_workspace(order, chunks):
    wl = W.get("image").with_(B=1, H=2)
    hq, hk, hv = _host_inputs(wl)
    s = P.Shape(wl.B, wl.H, wl.N, wl.d, wl.block)
    need = P.host_workspace_bytes(s, wl.topk, order, chunks=chunks)
    assert 0 < need <= P.STATIC_WORKSPACE_BYTES
    ref = P.pisa_host(hq, hk, hv, wl.block, wl.topk, order, wl.scale, chunks=chunks)
    for _ in range(2):
        got = P.pisa_host_static(hq, hk, hv, wl.block, wl.topk, order, wl.scale, chunks=chunks)
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    P.device_error()


def test_static_workspace_rejects_a_problem_too_large_for_it():
    wl = W.get("video").with_(H=2)
    s = P.Shape(wl.B, wl.H, wl.N, wl.d, wl.block)
    assert P.host_workspace_bytes(s, wl.topk, wl.order, chunks=1) > P.STATIC_WORKSPACE_BYTES
    q = torch.zeros((wl.B, wl.H, wl.N, wl.d), dtype=torch.bfloat16)
    with pytest.raises(P.PisaError, match="UNSUPPORTED"):
        P.pisa_host_static(q, q, q, wl.block, wl.topk, wl.order, wl.scale, chunks=1)

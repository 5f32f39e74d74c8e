"""The Python binding rejects mismatched buffers before anything reaches the library:
wrong shape, dtype or layout, a first-order statistic of the wrong order, index rows
of another block size, host tensors. Runs on the CPU; nothing is launched."""
import pytest

torch = pytest.importorskip("torch")

import block_sparse_attention_pisa_b200 as P  # noqa: E402
from block_sparse_attention_pisa_b200 import build as B  # noqa: E402

BF, F32, I32 = torch.bfloat16, torch.float32, torch.int32
Bn, H, N, d, b = 1, 2, 256, 128, 64
nB = N // b


@pytest.fixture(scope="module", autouse=True)
def _lib():
    B.build()
    P.lib()


def qkv():
    return [torch.zeros((Bn, H, N, d), dtype=BF) for _ in range(3)]


def stats(order=1):
    kbar = torch.zeros((Bn, H, nB, d), dtype=F32)
    S0 = torch.zeros_like(kbar)
    if order == 1:
        S1 = torch.zeros((Bn, H, nB, d, d), dtype=BF)
    elif order == 2:
        S1 = torch.zeros((Bn, H, d, d), dtype=F32)
    else:
        S1 = None
    return kbar, S0, S1


def idx(k=2, nb=nB):
    return torch.zeros((Bn, H, nb, k), dtype=I32)


def attn(**kw):
    Q, K, V = qkv()
    kbar, S0, S1 = stats(kw.pop("stat_order", kw.get("order", 1)))
    args = dict(Q=Q, K=K, V=V, kbar=kbar, S0=S0, S1=S1, idx=idx(), block=b, order=1, scale=0.1)
    args.update(kw)
    return P.attention(**args)


def test_valid_host_tensors_are_refused_as_host_tensors():
    with pytest.raises(ValueError, match="CUDA"):
        attn()
    Q, K, V = qkv()
    with pytest.raises(ValueError, match="CUDA"):
        P.block_stats(K, V, b, 1)
    with pytest.raises(ValueError, match="CUDA"):
        P.select(Q, stats()[0], b, 2)


@pytest.mark.parametrize("order", [1, 2])
def test_first_order_statistic_of_the_other_order(order):
    # per-block S1 passed at the hybrid order (or Hbar at order 1) would be read past its end
    with pytest.raises(ValueError, match="S1"):
        attn(order=order, stat_order=3 - order)


def test_index_rows_of_another_block_size():
    with pytest.raises(ValueError, match="idx"):
        attn(idx=idx(nb=nB // 2))
    with pytest.raises(ValueError, match="idx"):
        attn(idx=idx().to(torch.int64))


def test_statistics_of_another_block_size():
    kbar = torch.zeros((Bn, H, 2 * nB, d), dtype=F32)
    with pytest.raises(ValueError, match="kbar"):
        attn(kbar=kbar)
    with pytest.raises(ValueError, match="S0"):
        attn(S0=torch.zeros((Bn, H, nB, d), dtype=torch.float64))


def test_operand_dtypes_and_layout():
    Q, K, V = qkv()
    with pytest.raises(ValueError, match="K"):
        attn(K=K.float())
    with pytest.raises(ValueError, match="V"):
        attn(V=V[:, :, :N // 2])
    with pytest.raises(ValueError, match="O"):
        attn(out=torch.zeros((Bn, H, N, d), dtype=F32))
    t = torch.zeros((Bn, H, d, N), dtype=BF).transpose(-1, -2)
    with pytest.raises(ValueError, match="contiguous"):
        attn(K=t)
    with pytest.raises(ValueError, match="order"):
        attn(order=3)


def test_drop_ignores_statistics_and_zero_order_ignores_s1():
    # nothing is required of the statistics that the order does not read: the call gets as
    # far as the device check
    with pytest.raises(ValueError, match="CUDA"):
        attn(order=-1, kbar=None, S0=None, S1=None)
    with pytest.raises(ValueError, match="CUDA"):
        attn(order=0, S1=None)


def test_stats_and_select_outputs():
    Q, K, V = qkv()
    kbar, S0, S1 = stats(1)
    with pytest.raises(ValueError, match="S1"):
        P.block_stats(K, V, b, 2, out=(kbar, S0, S1))
    with pytest.raises(ValueError, match="kbar"):
        P.block_stats(K, V, b, 1, out=(kbar[:, :1], S0, S1))
    with pytest.raises(ValueError, match="V"):
        P.block_stats(K, V.float(), b, 1)
    with pytest.raises(ValueError, match="idx"):
        P.select(Q, kbar, b, 2, out=idx(k=3))
    with pytest.raises(ValueError, match="route"):
        P.select(Q, kbar, b, 2, route=torch.zeros((Bn, H, nB + 1), dtype=F32), lam=0.1)
    with pytest.raises(ValueError, match="kbar"):
        P.select(Q, kbar.double(), b, 2)


def test_routing_outputs():
    S1 = torch.zeros((Bn, H, nB, d, d), dtype=BF)
    with pytest.raises(ValueError, match="block count"):
        P.routing_norms(S1, b, N * 2)
    with pytest.raises(ValueError, match="M"):
        P.routing_norms(S1, b, N, out=(torch.zeros((Bn, H, d, d), dtype=F32), torch.zeros((Bn, H, nB + 1), dtype=F32)))
    with pytest.raises(ValueError, match="S1"):
        P.routing_norms(S1.float(), b, N)

"""Block selection with exact ties (GPU).

PISA explainer, technical summary section 2, "Covariance-aware routing": the critical
blocks of a query block are the top-k key blocks by pooled score, ties to the lower
block index. The parity tests excuse rows where the fp64 oracle sees a near-tie; here
every score is an exact small integer in fp32 and fp64 alike (each query block is made
of identical bf16 integer rows, so its mean is exact, and kbar holds small integers), so
ties are real and no row is excused: the GPU indices must equal the exact ranking (score
descending, block index ascending), kept in ascending block order.

Three score distributions exercise the selection's paths: integers spread over a wide
range (threshold bucket of one or a few keys), three distinct values (hundreds of keys
share the threshold value), and one value for every block (every key equal).
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_pisa_b200 as P

pytestmark = pytest.mark.gpu


def _exact_topk(scores, k):
    """[rows, nB] integer scores -> [rows, k] indices: k best, ties to the lower index,
    ascending."""
    order = np.lexsort((np.arange(scores.shape[1])[None, :].repeat(scores.shape[0], 0), -scores), axis=1)
    return np.sort(order[:, :k], axis=1)


def _case(B, H, nB, d, block, k, spread, seed):
    rng = np.random.default_rng(seed)
    # query block i of head h: `block` identical rows q_{h,i} with small integer entries
    qv = rng.integers(-spread, spread + 1, size=(B, H, nB, d)) if spread else np.ones((B, H, nB, d), np.int64)
    kb = rng.integers(-spread, spread + 1, size=(B, H, nB, d)) if spread else np.ones((B, H, nB, d), np.int64)
    if spread == 1:
        # three distinct scores per row: q in {0, 1}, kbar rows drawn from three patterns
        qv = np.ones((B, H, nB, d), np.int64)
        pat = np.stack([np.zeros(d), np.ones(d), 2 * np.ones(d)]).astype(np.int64)
        kb = pat[rng.integers(0, 3, size=(B, H, nB))]
    Q = np.repeat(qv, block, axis=2).astype(np.float32)           # [B, H, N, d], exact in bf16
    scores = np.einsum("bhid,bhjd->bhij", qv, kb)                  # exact integers
    exp = _exact_topk(scores.reshape(-1, nB), k).reshape(B, H, nB, k)
    dq = torch.from_numpy(Q).to(torch.bfloat16).cuda()
    dk = torch.from_numpy(kb.astype(np.float32)).cuda()
    return dq, dk, exp


@pytest.mark.parametrize("nB,d,block,k", [(512, 128, 64, 64), (591, 128, 128, 60), (64, 128, 64, 16),
                                          (128, 64, 128, 8), (4, 64, 64, 2), (300, 64, 64, 37)])
@pytest.mark.parametrize("spread", [40, 1, 0])
def test_exact_ties(nB, d, block, k, spread):
    dq, dk, exp = _case(1, 2, nB, d, block, k, spread, seed=nB * 7 + spread)
    assert float(dq.float().abs().max()) < 256 and torch.equal(dq.float(), dq.float().round())
    idx = P.select(dq, dk, block, k)
    torch.cuda.synchronize()
    P.device_error()
    got = idx.cpu().numpy()
    bad = np.argwhere(np.any(got != exp, axis=-1))
    assert bad.size == 0, f"{len(bad)} rows differ; first {bad[:3].tolist()}: {got[tuple(bad[0])][:8]} vs {exp[tuple(bad[0])][:8]}"

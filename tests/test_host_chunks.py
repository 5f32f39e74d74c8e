"""Host logic of the pipelined host entry point (CPU): the (batch, head) ranges."""
import pytest

import block_sparse_attention_pisa_b200 as P


@pytest.mark.parametrize("BH,chunks", [(24, 8), (24, 5), (3, 8), (1, 1), (48, 7), (40, 40)])
def test_head_chunks_cover_every_pair_once(BH, chunks):
    r = P.head_chunks(BH, chunks)
    assert r[0][0] == 0 and r[-1][1] == BH
    assert all(a < b for a, b in r)
    assert all(r[i][1] == r[i + 1][0] for i in range(len(r) - 1))
    assert len(r) == min(BH, chunks)
    sizes = [b - a for a, b in r]
    assert max(sizes) - min(sizes) <= 1

"""fp64 reference implementation of PISA (test infrastructure only).

Notation (PISA explainer, "PISA: Piecewise Sparse Attention Is Wiser for
Efficient Diffusion Transformers", technical summary section 2):

* tensors are [B, H, N, d]; block ``j`` holds tokens [j*b, min((j+1)*b, N))
  and has ``n_j`` real tokens (the last block may be ragged);
* for query block ``i`` the key/value blocks split into the critical set
  ``S_i`` (computed exactly) and the non-critical set ``U_i`` (approximated);
* ``x_t = scale * q_t`` is the scaled query of row ``t``;
* ``kbar_j`` is block j's mean key (the block centroid), ``S0_j`` its value
  sum, ``S1_j = sum_{n in j} (k_n - kbar_j) v_n^T`` (d x d, rows indexed by
  the key dimension, columns by the value dimension);
* ``alpha_{t,j} = exp(x_t . kbar_j)``.

The output is ``o_t = N_t / D_t`` with

    N_t = sum_{j in S_i} sum_n e^{x_t.k_{j,n}} v_{j,n}
        + sum_{j in U_i} alpha_{t,j} (S0_j + [order >= 1] S1_j^T x_t)
    D_t = sum_{j in S_i} sum_n e^{x_t.k_{j,n}} + sum_{j in U_i} n_j alpha_{t,j}

(section 2, "Core algorithm": the exact sparse term, the block zeroth-order
term with alpha defined from the block centroid, and a first-order term in the
third slot of the numerator; "Key insights": the approximations sit inside the
softmax numerator and denominator). The denominator's first-order part is
``x_t . sum_n (k_n - kbar_j) = 0`` identically and is therefore absent.
All exponents are shifted by the row maximum ``m_t`` before exponentiation;
the shift cancels in N_t / D_t.
"""
from __future__ import annotations

import numpy as np

NEAR_TIE_REL = 1e-5


def block_bounds(N: int, block: int):
    """[(start, end)] of every block; the last one may hold fewer than ``block`` tokens."""
    nB = -(-N // block)
    return [(j * block, min((j + 1) * block, N)) for j in range(nB)]


def block_stats(K, V, block: int, order: int = 1):
    """Block centroid, value sum and first-order matrix of every key/value block.

    Section 2, "Hardware implementation", precompute step (block centroids and
    value sums); the per-block first-order matrix is the Taylor term defined in
    the module docstring.

    Returns ``kbar`` [B,H,nB,d], ``S0`` [B,H,nB,d] and ``S1`` [B,H,nB,d,d]
    (``None`` when ``order == 0``), all float64.
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, N, d = K.shape
    bounds = block_bounds(N, block)
    nB = len(bounds)
    kbar = np.empty((B, H, nB, d))
    S0 = np.empty((B, H, nB, d))
    S1 = np.empty((B, H, nB, d, d)) if order >= 1 else None
    for j, (s, e) in enumerate(bounds):
        Kj = K[:, :, s:e, :]
        Vj = V[:, :, s:e, :]
        kbar[:, :, j] = Kj.sum(axis=2) / (e - s)
        S0[:, :, j] = Vj.sum(axis=2)
        if S1 is not None:
            centred = Kj - kbar[:, :, j][:, :, None, :]
            # S1[a, c] = sum_n centred[n, a] * v[n, c]
            S1[:, :, j] = np.matmul(np.swapaxes(centred, -1, -2), Vj)
    return kbar, S0, S1


def pooled_queries(Q, block: int):
    """Mean query of every query block (same partition as the key blocks)."""
    Q = np.asarray(Q, dtype=np.float64)
    B, H, N, d = Q.shape
    bounds = block_bounds(N, block)
    qbar = np.empty((B, H, len(bounds), d))
    for i, (s, e) in enumerate(bounds):
        qbar[:, :, i] = Q[:, :, s:e, :].sum(axis=2) / (e - s)
    return qbar


def select(Q, kbar, block: int, topk: int, route=None, lam: float = 0.0):
    """Top-k critical blocks of every query block.

    The page states that the critical blocks are the ones with the highest
    attention relevance (section 2, "Covariance-aware routing", first sentence).
    Relevance here is the pooled score ``qbar_i . kbar_j`` with ``qbar_i`` the
    mean query of block i. A positive softmax scale cannot change the order, so
    the scores are unscaled.

    Covariance-aware routing (same paragraph): with ``route`` = M [B,H,nB] (see
    ``routing_norms``) and a weight ``lam`` >= 0, the score of key block j is
    ``qbar_i . kbar_j + lam * M_j``, so that blocks whose first-order matrix
    departs most from the head's mean are favoured for exact treatment.

    Returns ``idx`` int32 [B,H,nB,topk] (each row ascending; ties between equal
    scores go to the lower block index), ``near_tie`` bool [B,H,nB] (the k-th
    and (k+1)-th scores agree to 1e-5 relative) and ``scores`` [B,H,nB,nB].
    """
    qbar = pooled_queries(Q, block)
    kbar = np.asarray(kbar, dtype=np.float64)
    B, H, nB, _ = qbar.shape
    if not (0 <= topk <= nB):
        raise ValueError("topk out of range")
    scores = np.matmul(qbar, np.swapaxes(kbar, -1, -2))
    if route is not None:
        scores = scores + lam * np.asarray(route, dtype=np.float64)[:, :, None, :]
    idx = np.empty((B, H, nB, topk), dtype=np.int32)
    near = np.zeros((B, H, nB), dtype=bool)
    cols = np.arange(nB)
    for b in range(B):
        for h in range(H):
            for i in range(nB):
                row = scores[b, h, i]
                # primary key: score descending; secondary key: block index ascending
                order = np.lexsort((cols, -row))
                idx[b, h, i] = np.sort(order[:topk])
                if 0 < topk < nB:
                    a, c = row[order[topk - 1]], row[order[topk]]
                    near[b, h, i] = abs(a - c) <= NEAR_TIE_REL * max(abs(a), abs(c))
    return idx, near, scores


def _top(row, count, among=None):
    """The `count` highest-scoring columns of `row` (restricted to `among` when given),
    equal scores resolved toward the lower column, returned ascending, plus the near-tie
    flag of the count-th / (count+1)-th place (within NEAR_TIE_REL relative)."""
    cols = np.arange(row.size) if among is None else np.asarray(among)
    vals = row[cols]
    order = np.lexsort((cols, -vals))
    near = False
    if 0 < count < cols.size:
        a, c = vals[order[count - 1]], vals[order[count]]
        near = abs(a - c) <= NEAR_TIE_REL * max(abs(a), abs(c))
    return np.sort(cols[order[:count]]), near


def select_grouped(Q, kbar, block: int, topk: int, group: int, candidates: int,
                   route=None, lam: float = 0.0):
    """Selection with one proxy query per group of query blocks.

    PIVOT page ("PIVOT slashes sparse-attention indexer cost 4x and cuts latency
    1.6x", gyaansetu), "Two observations behind PIVOT": neighbouring queries pick
    nearly the same top-k, so (1) g consecutive queries form a group, (2) their mean
    is the group's proxy query, (3) the indexer scores the proxy alone, and (4) the
    proxy's candidate list is refined for each member of the group; the reuse mode
    hands the proxy's list to every member unchanged.

    Here the indexer's units are query blocks: group m holds query blocks
    [m*group, min((m+1)*group, nB)), and its proxy is the mean of all real query rows
    of those blocks (the pooled query of the group). The proxy's `candidates` best key
    blocks by ``proxy . kbar_j (+ lam M_j)`` form the candidate list; each member query
    block i then keeps the `topk` candidates with the best ``qbar_i . kbar_j (+ lam
    M_j)``. `candidates` = topk is the reuse mode (the member step keeps every
    candidate); `candidates` = nB leaves only the member step, i.e. plain selection.
    Ties go to the lower block index; rows are ascending.

    Returns ``idx`` int32 [B,H,nB,topk] and ``near_tie`` bool [B,H,nB]: the row's
    proxy list or its member step had a near-tie at the cut (within 1e-5 relative).
    """
    Q = np.asarray(Q, dtype=np.float64)
    kbar = np.asarray(kbar, dtype=np.float64)
    B, H, N, d = Q.shape
    nB = kbar.shape[2]
    if not (1 <= topk <= candidates <= nB) or group < 1:
        raise ValueError("need 1 <= topk <= candidates <= nB and group >= 1")
    qbar = pooled_queries(Q, block)
    bias = np.zeros((B, H, nB)) if route is None else lam * np.asarray(route, dtype=np.float64)
    idx = np.empty((B, H, nB, topk), dtype=np.int32)
    near = np.zeros((B, H, nB), dtype=bool)
    span = group * block
    for b in range(B):
        for h in range(H):
            for m in range(-(-nB // group)):
                s, e = m * span, min((m + 1) * span, N)
                proxy = Q[b, h, s:e].sum(axis=0) / (e - s)
                cand, near_p = _top(kbar[b, h] @ proxy + bias[b, h], candidates)
                for i in range(m * group, min((m + 1) * group, nB)):
                    row = kbar[b, h] @ qbar[b, h, i] + bias[b, h]
                    idx[b, h, i], near_m = _top(row, topk, among=cand)
                    near[b, h, i] = near_p or near_m
    return idx, near


def round_to_bf16(x):
    """Round to the nearest bf16 value (ties to even) through fp32, as a value
    computed in fp32 and stored as bf16 is rounded."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def routing_norms(S1, stored_bf16: bool = True):
    """M_j = || H_j - Hbar ||_F for every block (section 2, "Covariance-aware
    routing": the norm of the block's deviation from the global first-order
    statistic; H_j is the block's first-order matrix S1_j and Hbar their mean
    over the head's blocks). The page writes a 2-norm without naming it; the
    Frobenius norm (the 2-norm of the matrix as a vector) is taken here.

    The norm feeds a top-k decision, so it is formed from S1 as it is stored
    for the kernels (fp32 values rounded to bf16) when ``stored_bf16``.
    Returns float64 [B,H,nB]."""
    S1 = np.asarray(S1, dtype=np.float64)
    if stored_bf16:
        S1 = round_to_bf16(S1)
    Hbar = S1.mean(axis=2)
    dev = S1 - Hbar[:, :, None]
    return np.sqrt((dev * dev).sum(axis=(-2, -1)))


def _query_blocks(nB, query_blocks):
    return range(nB) if query_blocks is None else query_blocks


ORDER_DROP, ORDER_ZERO, ORDER_FIRST, ORDER_HYBRID = -1, 0, 1, 2


def global_first_order(S1):
    """Hbar [B,H,d,d]: the mean of the per-block first-order matrices over all
    blocks of a head (section 2, "Core algorithm", global first-order correction;
    "Hardware implementation", precompute step)."""
    return np.asarray(S1, dtype=np.float64).mean(axis=2)


def attention(Q, K, V, kbar, S0, S1, idx, block: int, order: int, scale: float,
              query_blocks=None, heads=None):
    """PISA output rows (float64 [B,H,N,d]; rows of skipped query blocks are NaN).

    ``idx`` [B,H,nB,k] lists the critical blocks of each query block (any
    order; ``k`` may be 0). ``query_blocks`` / ``heads`` restrict the work to a
    sample; ``heads`` is a list of (b, h) pairs.

    ``order`` selects the treatment of the non-critical blocks:
      -1  drop them (keep-or-drop block-sparse attention, the baseline class the
          explainer contrasts with, section 1);
       0  zeroth-order Taylor term only;
       1  zeroth- plus per-block first-order term (``S1`` = per-block matrices);
       2  zeroth-order term plus the global first-order correction
          ``(x_t Hbar) sum_{j in U_i} alpha_{t,j}`` of section 2 ("Core
          algorithm": hybrid order), with ``S1`` = Hbar [B,H,d,d].
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, N, d = Q.shape
    bounds = block_bounds(N, block)
    nB = len(bounds)
    counts = np.array([e - s for s, e in bounds], dtype=np.float64)
    O = np.full((B, H, N, d), np.nan)
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in pairs:
        for i in _query_blocks(nB, query_blocks):
            s_i, e_i = bounds[i]
            X = scale * Q[b, h, s_i:e_i]                       # scaled queries of block i
            crit = sorted(set(int(j) for j in np.asarray(idx[b, h, i]).ravel()))
            crit_set = set(crit)
            rest = [j for j in range(nB) if j not in crit_set]
            # exact sparse term over every key of every critical block
            keys = [t for j in crit for t in range(*bounds[j])]
            z_ex = X @ K[b, h, keys].T                        # [n_i, |keys|]
            # zeroth-order exponents over the non-critical blocks
            z_ap = X @ kbar[b, h, rest].T                     # [n_i, |U|]
            if order == ORDER_DROP:
                z_ap = z_ap[:, :0]
                rest = []
            m = np.full(e_i - s_i, -np.inf)
            if z_ex.size:
                m = np.maximum(m, z_ex.max(axis=1))
            if z_ap.size:
                m = np.maximum(m, z_ap.max(axis=1))
            w = np.exp(z_ex - m[:, None])
            alpha = np.exp(z_ap - m[:, None])
            num = w @ V[b, h, keys] + alpha @ S0[b, h, rest]
            den = w.sum(axis=1) + alpha @ counts[rest]
            if order == ORDER_FIRST and rest:
                # S1_j^T x_t for every (j, t): first[j, t, c] = sum_a x[t, a] S1_j[a, c]
                first = np.matmul(X[None], S1[b, h, rest])
                num = num + np.einsum("tj,jtc->tc", alpha, first)
            elif order == ORDER_HYBRID and rest:
                # (x_t Hbar) scaled by the row's total non-critical weight
                num = num + (X @ S1[b, h]) * alpha.sum(axis=1)[:, None]
            O[b, h, s_i:e_i] = num / den[:, None]
    return O


def dense_attention(Q, K, V, scale: float):
    """Textbook softmax(scale Q K^T) V in float64."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    z = scale * np.matmul(Q, np.swapaxes(K, -1, -2))
    z = z - z.max(axis=-1, keepdims=True)
    p = np.exp(z)
    return np.matmul(p, V) / p.sum(axis=-1, keepdims=True)


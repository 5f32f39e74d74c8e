"""Pins of the CPU oracle against facts the method and the mathematics fix.

Each ``pin_*`` takes an oracle-like module (the real ``oracle`` package, or a
copy with a planted mistake) and returns a non-negative error; the test suite
asserts that the real oracle's errors are at round-off level and that every
planted mistake pushes at least one pin far above it.

None of these pins restates the oracle's vectorised formulas: they use scalar
brute force, exhaustive subset search, textbook softmax attention (scipy), a
second formulation of the first-order term, closed forms and convergence
rates.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
from scipy.special import softmax


def _rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------
# block statistics
# ----------------------------------------------------------------------------
def pin_stats_bruteforce(orc, seed=0):
    """Scalar loops over the definition of centroid, value sum and S1 (ragged N)."""
    r = _rng(seed)
    B, H, N, d, b = 1, 2, 11, 3, 4
    K = r.standard_normal((B, H, N, d))
    V = r.standard_normal((B, H, N, d))
    kbar, S0, S1 = orc.block_stats(K, V, b, order=1)
    err = 0.0
    for h in range(H):
        j = 0
        for start in range(0, N, b):
            toks = list(range(start, min(start + b, N)))
            cen = [sum(K[0, h, t, a] for t in toks) / len(toks) for a in range(d)]
            vs = [sum(V[0, h, t, c] for t in toks) for c in range(d)]
            for a in range(d):
                err = max(err, abs(kbar[0, h, j, a] - cen[a]))
                err = max(err, abs(S0[0, h, j, a] - vs[a]))
                for c in range(d):
                    ref = sum((K[0, h, t, a] - cen[a]) * V[0, h, t, c] for t in toks)
                    err = max(err, abs(S1[0, h, j, a, c] - ref))
            j += 1
    return err


def pin_stats_covariance(orc, seed=1):
    """With V = K, S1_j is n_j times the (biased) covariance of the block's keys."""
    r = _rng(seed)
    K = r.standard_normal((1, 1, 40, 5))
    _, _, S1 = orc.block_stats(K, K, 8, order=1)
    err = 0.0
    for j in range(5):
        ref = 8 * np.cov(K[0, 0, 8 * j:8 * j + 8].T, bias=True)
        err = max(err, np.abs(S1[0, 0, j] - ref).max())
    return err


def pin_stats_constant_values(orc, seed=2):
    """Constant value rows: S1 = 0 (centred keys sum to zero), S0 = n v."""
    r = _rng(seed)
    K = r.standard_normal((1, 1, 20, 4)) * 3 + 1
    V = np.broadcast_to(r.standard_normal(4), (1, 1, 20, 4)).copy()
    _, S0, S1 = orc.block_stats(K, V, 6, order=1)
    err = np.abs(S1).max()
    counts = [6, 6, 6, 2]
    for j, n in enumerate(counts):
        err = max(err, np.abs(S0[0, 0, j] - n * V[0, 0, 0]).max())
    return err


# ----------------------------------------------------------------------------
# selection
# ----------------------------------------------------------------------------
def _brute_select(qbar_row, kbar, k):
    """Subset of size k with the largest total score; ties -> lexicographically smallest."""
    nB = kbar.shape[0]
    sc = [sum(qbar_row[a] * kbar[j, a] for a in range(kbar.shape[1])) for j in range(nB)]
    best, best_set = -math.inf, None
    for sub in itertools.combinations(range(nB), k):      # lexicographic order
        tot = sum(sc[j] for j in sub)
        if tot > best + 1e-12:
            best, best_set = tot, sub
    return list(best_set)


def pin_select_bruteforce(orc, seed=3, trials=30):
    """Exhaustive subset search on 4-8 blocks, ragged N included. Returns #mismatches."""
    r = _rng(seed)
    bad = 0
    for t in range(trials):
        b = int(r.integers(1, 5))
        nB = int(r.integers(4, 9))
        N = b * nB - int(r.integers(0, b))
        nB = -(-N // b)
        d = int(r.integers(1, 5))
        k = int(r.integers(1, nB + 1))
        Q = r.standard_normal((1, 1, N, d))
        kbar = r.standard_normal((1, 1, nB, d))
        if t % 3 == 0:            # plant exact ties: duplicate some centroids
            kbar[0, 0, nB - 1] = kbar[0, 0, 0]
            kbar[0, 0, nB // 2] = kbar[0, 0, 1]
        idx, _, _ = orc.select(Q, kbar, b, k)
        for i in range(nB):
            rows = [s for s in range(i * b, min(i * b + b, N))]
            qbar = [sum(Q[0, 0, s, a] for s in rows) / len(rows) for a in range(d)]
            ref = _brute_select(qbar, kbar[0, 0], k)
            if list(idx[0, 0, i]) != ref:
                bad += 1
    return bad


def pin_select_ties(orc):
    """All centroids equal: every row must take blocks 0..k-1 (lower index wins)."""
    Q = _rng(4).standard_normal((1, 1, 32, 3))
    kbar = np.ones((1, 1, 8, 3))
    idx, _, _ = orc.select(Q, kbar, 4, 3)
    return int(np.any(idx != np.arange(3)))


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------
def _textbook(Q, K, V, scale):
    """softmax(scale Q K^T) V with scipy's softmax (independent of the oracle's)."""
    z = scale * np.einsum("bhqd,bhkd->bhqk", Q, K)
    return np.einsum("bhqk,bhkd->bhqd", softmax(z, axis=-1), V)


def _full_idx(B, H, nB, k=None):
    k = nB if k is None else k
    return np.broadcast_to(np.arange(k, dtype=np.int32), (B, H, nB, k)).copy()


def pin_dense_textbook(orc, seed=21):
    """oracle.dense_attention against scipy's softmax, scalar loops on a tiny case, and
    large logit offsets (a per-row shift of the logits cannot change a softmax)."""
    r = _rng(seed)
    B, H, N, M, d = 1, 2, 9, 13, 5
    Q = r.standard_normal((B, H, N, d))
    K = r.standard_normal((B, H, M, d))
    V = r.standard_normal((B, H, M, d))
    scale = 0.7
    err = float(np.abs(orc.dense_attention(Q, K, V, scale) - _textbook(Q, K, V, scale)).max())
    # one row written out with scalar loops
    out = orc.dense_attention(Q, K, V, scale)
    for h in range(H):
        for t in (0, N - 1):
            z = [scale * sum(Q[0, h, t, a] * K[0, h, n, a] for a in range(d)) for n in range(M)]
            w = [math.exp(v - max(z)) for v in z]
            for c in range(d):
                ref = sum(w[n] * V[0, h, n, c] for n in range(M)) / sum(w)
                err = max(err, abs(out[0, h, t, c] - ref))
    # logits near 700 overflow exp() unless the row maximum is taken out first; the
    # rows get different offsets (q_t -> q_t + s_t u with u . k_n = const over n)
    u = np.zeros(d)
    u[0] = 1.0
    K2 = K.copy()
    K2[..., 0] = 50.0
    Q2 = Q + (np.arange(N) * 2.0 + 14.0)[None, None, :, None] * u
    err = max(err, float(np.abs(orc.dense_attention(Q2, K2, V, 1.0)
                                - _textbook(Q2 - Q2[..., :1] * u, K2, V, 1.0)).max()))
    return err


def pin_all_selected_is_dense(orc, seed=5):
    r = _rng(seed)
    B, H, N, d, b = 1, 2, 45, 8, 8           # ragged last block
    Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
    kbar, S0, S1 = orc.block_stats(K, V, b)
    nB = -(-N // b)
    out = orc.attention(Q, K, V, kbar, S0, S1, _full_idx(B, H, nB), b, 1, 0.4)
    return np.abs(out - _textbook(Q, K, V, 0.4)).max()


def pin_block_one_is_exact(orc, seed=6):
    """Block size 1: kbar = k and S1 = 0, so any selection gives dense attention."""
    r = _rng(seed)
    B, H, N, d = 1, 1, 24, 4
    Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
    kbar, S0, S1 = orc.block_stats(K, V, 1)
    idx = np.stack([r.choice(N, 5, replace=False) for _ in range(N)])[None, None].astype(np.int32)
    err = 0.0
    for order in (0, 1):
        out = orc.attention(Q, K, V, kbar, S0, S1, idx, 1, order, 0.7)
        err = max(err, np.abs(out - _textbook(Q, K, V, 0.7)).max())
    return err


def pin_identical_keys_exact(orc, seed=7):
    """A block of identical keys is exact at order 0 (and order 1, where S1 = 0)."""
    r = _rng(seed)
    B, H, N, d, b = 1, 1, 48, 6, 8
    c = r.standard_normal((N // b, d))
    K = np.repeat(c, b, axis=0)[None, None]
    Q, V = (r.standard_normal((B, H, N, d)) for _ in range(2))
    kbar, S0, S1 = orc.block_stats(K, V, b)
    idx = np.full((1, 1, N // b, 1), 2, dtype=np.int32)
    err = 0.0
    for order in (0, 1):
        out = orc.attention(Q, K, V, kbar, S0, S1, idx, b, order, 0.5)
        err = max(err, np.abs(out - _textbook(Q, K, V, 0.5)).max())
    return err


def convergence_slopes(orc, seed=8):
    """log-log slopes of the error vs dense as the in-block key spread eps shrinks."""
    r = _rng(seed)
    B, H, N, d, b = 1, 1, 64, 8, 8
    nB = N // b
    c = r.standard_normal((nB, d))
    z = r.standard_normal((N, d))
    Q = r.standard_normal((B, H, N, d))
    V = r.standard_normal((B, H, N, d))
    idx = np.zeros((1, 1, nB, 1), dtype=np.int32)
    epss = [0.4, 0.2, 0.1, 0.05]
    errs = {0: [], 1: []}
    for eps in epss:
        K = (np.repeat(c, b, axis=0) + eps * z)[None, None]
        kbar, S0, S1 = orc.block_stats(K, V, b)
        ref = _textbook(Q, K, V, 0.5)
        for order in (0, 1):
            out = orc.attention(Q, K, V, kbar, S0, S1, idx, b, order, 0.5)
            errs[order].append(np.abs(out - ref).max())
    le = np.log(epss)
    return {o: float(np.polyfit(le, np.log(errs[o]), 1)[0]) for o in (0, 1)}


def pin_order0_pseudo_tokens(orc, seed=9):
    """No critical block, order 0: softmax over pseudo-tokens (kbar_j, S0_j/n_j) with a
    log-count bias ln n_j (textbook softmax attention over pooled tokens)."""
    r = _rng(seed)
    B, H, N, d, b = 1, 1, 30, 5, 7          # counts 7,7,7,7,2
    Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
    kbar, S0, S1 = orc.block_stats(K, V, b)
    nB = -(-N // b)
    idx = np.zeros((1, 1, nB, 0), dtype=np.int32)
    out = orc.attention(Q, K, V, kbar, S0, S1, idx, b, 0, 0.9)
    counts = np.array([min(N, (j + 1) * b) - j * b for j in range(nB)], dtype=float)
    z = 0.9 * Q[0, 0] @ kbar[0, 0].T + np.log(counts)[None, :]
    ref = softmax(z, axis=-1) @ (S0[0, 0] / counts[:, None])
    return np.abs(out[0, 0] - ref).max()


def pin_first_order_key_form(orc, seed=10):
    """Order-1 output from a second formulation: S1_j^T x = sum_n (x.(k_n - kbar_j)) v_n,
    i.e. each non-critical key gets weight e^{x.kbar}(1 + x.(k - kbar))."""
    r = _rng(seed)
    B, H, N, d, b = 1, 2, 40, 6, 8
    Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
    kbar, S0, S1 = orc.block_stats(K, V, b)
    nB = N // b
    idx = np.stack([np.sort(r.choice(nB, 2, replace=False)) for _ in range(B * H * nB)])
    idx = idx.reshape(B, H, nB, 2).astype(np.int32)
    scale = 0.6
    out = orc.attention(Q, K, V, kbar, S0, S1, idx, b, 1, scale)
    err = 0.0
    for h in range(H):
        for i in range(nB):
            crit = set(idx[0, h, i].tolist())
            for t in range(i * b, i * b + b):
                x = scale * Q[0, h, t]
                wts, vals = [], []
                for j in range(nB):
                    kb = K[0, h, j * b:j * b + b].mean(axis=0)
                    for n in range(j * b, j * b + b):
                        if j in crit:
                            wts.append(math.exp(x @ K[0, h, n]))
                        else:
                            wts.append(math.exp(x @ kb) * (1.0 + x @ (K[0, h, n] - kb)))
                        vals.append(V[0, h, n])
                # the denominator of a non-critical block is n_j e^{x.kbar}: the
                # first-order weights sum to that exactly
                ref = np.array(wts) @ np.array(vals) / sum(wts)
                err = max(err, np.abs(out[0, h, t] - ref).max())
    return err


def pin_linear_in_values(orc, seed=11):
    r = _rng(seed)
    B, H, N, d, b = 1, 1, 32, 4, 8
    Q, K, V1, V2 = (r.standard_normal((B, H, N, d)) for _ in range(4))
    idx = np.array([[[[1], [0], [3], [2]]]], dtype=np.int32)

    def run(V):
        kb, s0, s1 = orc.block_stats(K, V, b)
        return orc.attention(Q, K, V, kb, s0, s1, idx, b, 1, 0.5)
    return np.abs(run(2.0 * V1 - 3.0 * V2) - (2.0 * run(V1) - 3.0 * run(V2))).max()


def pin_permutation_in_block(orc, seed=12):
    """Permuting (k, v) pairs inside a non-critical block leaves the output unchanged."""
    r = _rng(seed)
    B, H, N, d, b = 1, 1, 32, 4, 8
    Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
    idx = np.zeros((1, 1, 4, 1), dtype=np.int32)
    perm = np.arange(N)
    perm[16:24] = 16 + r.permutation(8)
    outs = []
    for P in (np.arange(N), perm):
        Kp, Vp = K[:, :, P], V[:, :, P]
        kb, s0, s1 = orc.block_stats(Kp, Vp, b)
        outs.append(orc.attention(Q, Kp, Vp, kb, s0, s1, idx, b, 1, 0.5))
    return np.abs(outs[0] - outs[1]).max()


def pin_order0_convex(orc, seed=13):
    """Order 0 is a convex combination of exact values and block mean values:
    returns the largest violation of min <= o <= max (per coordinate)."""
    r = _rng(seed)
    B, H, N, d, b = 1, 1, 40, 4, 8
    Q, K, V = (r.standard_normal((B, H, N, d)) * 2 for _ in range(3))
    kb, s0, s1 = orc.block_stats(K, V, b)
    idx = np.array([[[[0], [1], [2], [3], [4]]]], dtype=np.int32)
    out = orc.attention(Q, K, V, kb, s0, s1, idx, b, 0, 1.0)
    pool = np.concatenate([V[0, 0], s0[0, 0] / b], axis=0)
    lo, hi = pool.min(axis=0), pool.max(axis=0)
    return float(max(0.0, (lo - out[0, 0]).max(), (out[0, 0] - hi).max()))


def pin_worked_example(orc, case):
    """Scalar (d = 1) worked example expanded by hand (tests/golden/worked_example.json)."""
    q, k, v = (np.array(case[n], dtype=float) for n in ("q", "k", "v"))
    b, scale = case["block"], case["scale"]
    crit = case["critical"]                  # one list per query block
    N = len(q)
    Q, K, V = (a.reshape(1, 1, N, 1) for a in (q, k, v))
    kb, s0, s1 = orc.block_stats(K, V, b)
    idx = np.array(crit, dtype=np.int32).reshape(1, 1, len(crit), -1)
    err = 0.0
    for order in (0, 1):
        out = orc.attention(Q, K, V, kb, s0, s1, idx, b, order, scale)
        for t in range(N):
            x = scale * q[t]
            num = den = 0.0
            for j in range(-(-N // b)):
                toks = range(j * b, min(j * b + b, N))
                if j in crit[t // b]:
                    for n in toks:
                        num += math.exp(x * k[n]) * v[n]
                        den += math.exp(x * k[n])
                else:
                    kbar = sum(k[n] for n in toks) / len(toks)
                    vsum = sum(v[n] for n in toks)
                    first = sum((k[n] - kbar) * v[n] for n in toks)
                    a = math.exp(x * kbar)
                    num += a * (vsum + (order * first * x))
                    den += a * len(toks)
            err = max(err, abs(out[0, 0, t, 0] - num / den))
    return err


# ----------------------------------------------------------------------------
# keep-or-drop and hybrid order
# ----------------------------------------------------------------------------
def pin_drop_is_masked_softmax(orc, seed=14):
    """Keep-or-drop: textbook softmax over the critical blocks' keys only (the
    other logits masked to -inf), ragged last block included."""
    r = _rng(seed)
    B, H, N, d, b = 1, 2, 37, 5, 8
    Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
    kbar, S0, S1 = orc.block_stats(K, V, b)
    nB = -(-N // b)
    idx = np.stack([np.sort(r.choice(nB, 2, replace=False)) for _ in range(B * H * nB)])
    idx = idx.reshape(B, H, nB, 2).astype(np.int32)
    out = orc.attention(Q, K, V, kbar, S0, S1, idx, b, -1, 0.7)
    err = 0.0
    for h in range(H):
        z = 0.7 * Q[0, h] @ K[0, h].T
        for t in range(N):
            keep = np.zeros(N, dtype=bool)
            for j in idx[0, h, t // b]:
                keep[j * b:min(j * b + b, N)] = True
            zt = np.where(keep, z[t], -np.inf)
            err = max(err, np.abs(softmax(zt) @ V[0, h] - out[0, h, t]).max())
    return err


def pin_hybrid_bruteforce(orc, seed=15):
    """Hybrid order written out with scalar loops: Hbar = mean over all blocks of
    sum_n (k_n - kbar_j) v_n^T, then N_t = exact + sum_U alpha (sum v) +
    (x Hbar) sum_U alpha, D_t = exact + sum_U n_j alpha (ragged last block)."""
    r = _rng(seed)
    B, H, N, d, b = 1, 1, 27, 3, 6
    Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
    kbar, S0, S1 = orc.block_stats(K, V, b)
    Hbar = orc.global_first_order(S1)
    nB = -(-N // b)
    blocks = [list(range(j * b, min(j * b + b, N))) for j in range(nB)]
    cen = [[sum(K[0, 0, n, a] for n in bl) / len(bl) for a in range(d)] for bl in blocks]
    ref_H = [[sum(sum((K[0, 0, n, a] - cen[j][a]) * V[0, 0, n, c] for n in bl)
                  for j, bl in enumerate(blocks)) / nB for c in range(d)] for a in range(d)]
    err = float(np.abs(Hbar[0, 0] - np.array(ref_H)).max())
    crit = [[i, (i + 2) % nB] for i in range(nB)]
    idx = np.sort(np.array(crit, dtype=np.int32), axis=1)[None, None]
    scale = 0.8
    out = orc.attention(Q, K, V, kbar, S0, Hbar, idx, b, 2, scale)
    for t in range(N):
        x = [scale * Q[0, 0, t, a] for a in range(d)]
        num = [0.0] * d
        den = 0.0
        asum = 0.0
        for j, bl in enumerate(blocks):
            if j in crit[t // b]:
                for n in bl:
                    w = math.exp(sum(x[a] * K[0, 0, n, a] for a in range(d)))
                    den += w
                    for c in range(d):
                        num[c] += w * V[0, 0, n, c]
            else:
                al = math.exp(sum(x[a] * cen[j][a] for a in range(d)))
                asum += al
                den += len(bl) * al
                for c in range(d):
                    num[c] += al * sum(V[0, 0, n, c] for n in bl)
        for c in range(d):
            num[c] += asum * sum(x[a] * ref_H[a][c] for a in range(d))
            err = max(err, abs(out[0, 0, t, c] - num[c] / den))
    return err


def pin_hybrid_shared_first_order(orc, seed=16):
    """Blocks that are translated copies of one pattern (k = c_j + z_n, v = u_n)
    share a single first-order matrix, so Hbar = S1_j and the hybrid order equals
    the per-block first-order output."""
    r = _rng(seed)
    B, H, b, nB, d = 1, 1, 8, 6, 5
    N = b * nB
    c = r.standard_normal((nB, d)) * 2
    z = r.standard_normal((b, d)) * 0.3
    u = r.standard_normal((b, d))
    K = (np.repeat(c, b, axis=0) + np.tile(z, (nB, 1)))[None, None]
    V = np.tile(u, (nB, 1))[None, None]
    Q = r.standard_normal((B, H, N, d))
    kbar, S0, S1 = orc.block_stats(K, V, b)
    idx = np.array([[[[i] for i in range(nB)]]], dtype=np.int32)
    first = orc.attention(Q, K, V, kbar, S0, S1, idx, b, 1, 0.6)
    hybrid = orc.attention(Q, K, V, kbar, S0, orc.global_first_order(S1), idx, b, 2, 0.6)
    return float(np.abs(first - hybrid).max())


def pin_hybrid_all_selected_is_dense(orc, seed=17):
    r = _rng(seed)
    B, H, N, d, b = 1, 1, 30, 4, 8
    Q, K, V = (r.standard_normal((B, H, N, d)) for _ in range(3))
    kbar, S0, S1 = orc.block_stats(K, V, b)
    nB = -(-N // b)
    out = orc.attention(Q, K, V, kbar, S0, orc.global_first_order(S1), _full_idx(B, H, nB), b, 2, 0.5)
    return np.abs(out - _textbook(Q, K, V, 0.5)).max()


# ----------------------------------------------------------------------------
# covariance-aware routing
# ----------------------------------------------------------------------------
def pin_round_to_bf16(orc, seed=18):
    """Nearest bf16 by enumeration of the neighbouring bf16 values (ties to the
    even mantissa), on random fp32 values and on planted halfway cases."""
    r = _rng(seed)
    x = (r.standard_normal(400) * np.exp(r.uniform(-20, 20, 400))).astype(np.float32)
    half = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.0 - 2.0 ** -7, 3.0 + 2.0 ** -7], dtype=np.float32)
    x = np.concatenate([x, half])
    got = orc.round_to_bf16(x.astype(np.float64))
    bad = 0
    for v, g in zip(x.tolist(), got.tolist()):
        bits = int(np.array(v, dtype=np.float32).view(np.uint32))
        lo = bits & 0xFFFF0000                     # truncation toward zero (same sign)
        hi = lo + 0x10000                          # next bf16 away from zero
        cand = [float(np.array(c, dtype=np.uint32).view(np.float32)) for c in (lo, hi)]
        dl, dh = abs(v - cand[0]), abs(v - cand[1])
        if dl < dh or (dl == dh and ((lo >> 16) & 1) == 0):
            ref = cand[0]
        else:
            ref = cand[1]
        bad += g != ref
    return bad


def pin_routing_norms_bruteforce(orc, seed=19):
    """M_j = sqrt(sum_{a,c} (S1_j[a,c] - Hbar[a,c])^2) by scalar loops; the inputs are
    bf16 values already, so the stored-precision rounding is the identity."""
    r = _rng(seed)
    nB, d = 5, 3
    S1 = orc.round_to_bf16(r.standard_normal((1, 2, nB, d, d)) * 3)
    M = orc.routing_norms(S1)
    err = 0.0
    for h in range(2):
        mean = [[sum(S1[0, h, k, a, c] for k in range(nB)) / nB for c in range(d)] for a in range(d)]
        for j in range(nB):
            ref = math.sqrt(sum((S1[0, h, j, a, c] - mean[a][c]) ** 2 for a in range(d) for c in range(d)))
            err = max(err, abs(M[0, h, j] - ref))
    return err


def pin_routed_select_bruteforce(orc, seed=20, trials=30):
    """Exhaustive subset search over the scores qbar . kbar_j + lam * M_j (ragged N,
    planted ties). Returns #mismatches."""
    r = _rng(seed)
    bad = 0
    for t in range(trials):
        b = int(r.integers(1, 5))
        nB = int(r.integers(4, 9))
        N = b * nB - int(r.integers(0, b))
        nB = -(-N // b)
        d = int(r.integers(1, 4))
        k = int(r.integers(1, nB + 1))
        lam = float(r.uniform(0.1, 3.0))
        Q = r.standard_normal((1, 1, N, d))
        kbar = r.standard_normal((1, 1, nB, d))
        M = np.abs(r.standard_normal((1, 1, nB)))
        if t % 3 == 0:            # ties: two blocks with equal centroid and equal norm
            kbar[0, 0, nB - 1] = kbar[0, 0, 0]
            M[0, 0, nB - 1] = M[0, 0, 0]
        idx, _, _ = orc.select(Q, kbar, b, k, route=M, lam=lam)
        for i in range(nB):
            rows = list(range(i * b, min(i * b + b, N)))
            qbar = [sum(Q[0, 0, s, a] for s in rows) / len(rows) for a in range(d)]
            sc = [sum(qbar[a] * kbar[0, 0, j, a] for a in range(d)) + lam * M[0, 0, j] for j in range(nB)]
            best, best_set = -math.inf, None
            for sub in itertools.combinations(range(nB), k):
                tot = sum(sc[j] for j in sub)
                if tot > best + 1e-12:
                    best, best_set = tot, sub
            bad += list(idx[0, 0, i]) != list(best_set)
    return bad


# ----------------------------------------------------------------------------
# selection amortisation: one proxy query per group of query blocks
# ----------------------------------------------------------------------------
def _best_subset(scores, among, k):
    """Subset of `among` (size k) with the largest total score; ties -> the
    lexicographically smallest subset (itertools.combinations order)."""
    best, best_set = -math.inf, None
    for sub in itertools.combinations(sorted(among), k):
        tot = sum(scores[j] for j in sub)
        if tot > best + 1e-12:
            best, best_set = tot, sub
    return list(best_set)


def pin_grouped_bruteforce(orc, seed=22, trials=24):
    """Grouped selection by scalar loops: the proxy is the mean of every real query row
    of the group, its candidate list the best `c` blocks by exhaustive subset search,
    and each member's row the best `k` of those candidates for its own pooled query
    (ragged N, planted ties, optional routing bias). Returns #mismatched rows."""
    r = _rng(seed)
    bad = 0
    for t in range(trials):
        b = int(r.integers(1, 4))
        nB = int(r.integers(4, 9))
        N = b * nB - int(r.integers(0, b))
        nB = -(-N // b)
        d = int(r.integers(1, 4))
        g = int(r.integers(1, 4))
        k = int(r.integers(1, nB + 1))
        c = int(r.integers(k, nB + 1))
        Q = r.standard_normal((1, 1, N, d))
        kbar = r.standard_normal((1, 1, nB, d))
        if t % 3 == 0:
            kbar[0, 0, nB - 1] = kbar[0, 0, 0]
        lam = float(r.uniform(0.2, 2.0)) if t % 2 else 0.0
        M = np.abs(r.standard_normal((1, 1, nB)))
        idx, _ = orc.select_grouped(Q, kbar, b, k, g, c, route=M if lam else None, lam=lam)
        bias = [lam * M[0, 0, j] for j in range(nB)]
        for m in range(-(-nB // g)):
            rows = list(range(m * g * b, min((m + 1) * g * b, N)))
            proxy = [sum(Q[0, 0, s, a] for s in rows) / len(rows) for a in range(d)]
            psc = [sum(proxy[a] * kbar[0, 0, j, a] for a in range(d)) + bias[j] for j in range(nB)]
            cand = _best_subset(psc, range(nB), c)
            for i in range(m * g, min((m + 1) * g, nB)):
                qrows = list(range(i * b, min(i * b + b, N)))
                qb = [sum(Q[0, 0, s, a] for s in qrows) / len(qrows) for a in range(d)]
                msc = [sum(qb[a] * kbar[0, 0, j, a] for a in range(d)) + bias[j] for j in range(nB)]
                bad += list(idx[0, 0, i]) != _best_subset(msc, cand, k)
    return bad


def pin_grouped_special_cases(orc, seed=23):
    """Group 1 with any candidate count, and any group with candidates = nB, reduce to
    plain selection; candidates = topk (the reuse mode) gives every member of a group
    the same row. Returns #violations."""
    r = _rng(seed)
    B, H, N, d, b = 1, 2, 77, 5, 6
    nB = -(-N // b)
    Q = r.standard_normal((B, H, N, d))
    kbar = r.standard_normal((B, H, nB, d))
    plain, _, _ = orc.select(Q, kbar, b, 4)
    bad = 0
    for c in (4, 7, nB):
        bad += int(np.any(orc.select_grouped(Q, kbar, b, 4, 1, c)[0] != plain))
    for g in (2, 3, 5):
        bad += int(np.any(orc.select_grouped(Q, kbar, b, 4, g, nB)[0] != plain))
        reuse, _ = orc.select_grouped(Q, kbar, b, 4, g, 4)
        for m in range(-(-nB // g)):
            members = reuse[:, :, m * g:min((m + 1) * g, nB)]
            bad += int(np.any(members != members[:, :, :1]))
    return bad

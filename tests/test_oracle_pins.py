"""The CPU oracle against what the method and the mathematics fix (no GPU).

Also plants plausible mistakes in copies of the oracle (source mutations, on
the CPU) and checks that at least one pin catches each of them.
"""
import json
import os
import types

import numpy as np
import pytest

import oracle
from tests import oracle_pins as P

HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE_SRC = os.path.join(os.path.dirname(HERE), "oracle", "pisa.py")
EXAMPLE = json.load(open(os.path.join(HERE, "golden", "worked_example.json")))

TOL = 1e-10


def _pins(orc):
    """name -> (value, passes?) for every pin."""
    out = {}
    for name, fn, ok in [
        ("stats_bruteforce", P.pin_stats_bruteforce, lambda e: e < TOL),
        ("stats_covariance", P.pin_stats_covariance, lambda e: e < TOL),
        ("stats_constant_values", P.pin_stats_constant_values, lambda e: e < TOL),
        ("select_bruteforce", P.pin_select_bruteforce, lambda e: e == 0),
        ("select_ties", P.pin_select_ties, lambda e: e == 0),
        ("dense_textbook", P.pin_dense_textbook, lambda e: e < TOL),
        ("all_selected_is_dense", P.pin_all_selected_is_dense, lambda e: e < TOL),
        ("block_one_is_exact", P.pin_block_one_is_exact, lambda e: e < TOL),
        ("identical_keys_exact", P.pin_identical_keys_exact, lambda e: e < TOL),
        ("order0_pseudo_tokens", P.pin_order0_pseudo_tokens, lambda e: e < TOL),
        ("first_order_key_form", P.pin_first_order_key_form, lambda e: e < TOL),
        ("linear_in_values", P.pin_linear_in_values, lambda e: e < TOL),
        ("permutation_in_block", P.pin_permutation_in_block, lambda e: e < TOL),
        ("order0_convex", P.pin_order0_convex, lambda e: e <= 1e-12),
        ("worked_example", lambda o: P.pin_worked_example(o, EXAMPLE), lambda e: e < TOL),
        ("drop_is_masked_softmax", P.pin_drop_is_masked_softmax, lambda e: e < TOL),
        ("hybrid_bruteforce", P.pin_hybrid_bruteforce, lambda e: e < TOL),
        ("hybrid_shared_first_order", P.pin_hybrid_shared_first_order, lambda e: e < TOL),
        ("hybrid_all_selected_is_dense", P.pin_hybrid_all_selected_is_dense, lambda e: e < TOL),
        ("round_to_bf16", P.pin_round_to_bf16, lambda e: e == 0),
        ("routing_norms_bruteforce", P.pin_routing_norms_bruteforce, lambda e: e < TOL),
        ("routed_select_bruteforce", P.pin_routed_select_bruteforce, lambda e: e == 0),
        ("grouped_bruteforce", P.pin_grouped_bruteforce, lambda e: e == 0),
        ("grouped_special_cases", P.pin_grouped_special_cases, lambda e: e == 0),
    ]:
        try:
            v = fn(orc)
            out[name] = (v, bool(ok(v)))
        except Exception as exc:  # a mutant may crash a pin: that counts as caught
            out[name] = (repr(exc), False)
    slopes = P.convergence_slopes(orc)
    out["convergence_order0"] = (slopes[0], 0.8 < slopes[0] < 1.3)
    out["convergence_order1"] = (slopes[1], 1.7 < slopes[1] < 2.4)
    return out


@pytest.fixture(scope="module")
def real_pins():
    return _pins(oracle)


@pytest.mark.parametrize("name", [
    "stats_bruteforce", "stats_covariance", "stats_constant_values", "select_bruteforce",
    "select_ties", "dense_textbook", "all_selected_is_dense", "block_one_is_exact", "identical_keys_exact",
    "order0_pseudo_tokens", "first_order_key_form", "linear_in_values",
    "permutation_in_block", "order0_convex", "worked_example",
    "convergence_order0", "convergence_order1", "drop_is_masked_softmax", "hybrid_bruteforce",
    "hybrid_shared_first_order", "hybrid_all_selected_is_dense", "round_to_bf16",
    "routing_norms_bruteforce", "routed_select_bruteforce", "grouped_bruteforce",
    "grouped_special_cases"])
def test_pin(real_pins, name):
    value, ok = real_pins[name]
    assert ok, f"{name}: {value}"


def test_near_tie_flag():
    """Two centroids whose scores differ by 1e-7 relative straddle the k-th place."""
    Q = np.ones((1, 1, 16, 2))
    kbar = np.array([[[[3.0, 0.0], [1.0, 0.0], [1.0 + 1e-7, 0.0], [0.0, 0.0]]]])
    idx, near, _ = oracle.select(Q, kbar, 4, 2)
    assert list(idx[0, 0, 0]) == [0, 2] and near[0, 0, 0]
    idx, near, _ = oracle.select(Q, kbar, 4, 1)
    assert list(idx[0, 0, 0]) == [0] and not near[0, 0, 0]


MUTATIONS = {
    "S1 transposed in stats": ("np.swapaxes(centred, -1, -2), Vj", "np.swapaxes(Vj, -1, -2), centred"),
    "count dropped from denominator": ("alpha @ counts[rest]", "alpha.sum(axis=1)"),
    "ties to the higher index": ("np.lexsort((cols, -row))", "np.lexsort((-cols, -row))"),
    "lowest scores selected": ("np.lexsort((cols, -row))", "np.lexsort((cols, row))"),
    "scale missing from alpha": ("z_ap = X @ kbar", "z_ap = Q[b, h, s_i:e_i] @ kbar"),
    "first-order sign flipped": ("num = num + np.einsum", "num = num - np.einsum"),
    "ragged centroid over b": ("Kj.sum(axis=2) / (e - s)", "Kj.sum(axis=2) / block"),
    "S1 transposed in attention": ("np.matmul(X[None], S1[b, h, rest])",
                                   "np.matmul(X[None], np.swapaxes(S1[b, h, rest], -1, -2))"),
    "value mean instead of sum": ("S0[:, :, j] = Vj.sum(axis=2)", "S0[:, :, j] = Vj.mean(axis=2)"),
    "pooled query over wrong rows": ("Q[:, :, s:e, :].sum(axis=2) / (e - s)",
                                     "Q[:, :, s:s + 1, :].sum(axis=2)"),
    "exact keys from the wrong block": ("for t in range(*bounds[j])]", "for t in range(*bounds[(j + 1) % nB])]"),
    "drop keeps the zeroth-order terms": ("z_ap = z_ap[:, :0]", "z_ap = z_ap"),
    "Hbar summed instead of averaged": ("mean(axis=2)", "sum(axis=2)"),
    "Hbar transposed": ("(X @ S1[b, h])", "(X @ S1[b, h].T)"),
    "hybrid weight from all blocks": ("* alpha.sum(axis=1)[:, None]",
                                      "* (alpha.sum(axis=1) + w.sum(axis=1))[:, None]"),
    "hybrid term dropped": ("num = num + (X @ S1[b, h])", "num = num + 0 * (X @ S1[b, h])"),
    "routing norm not centred": ("dev = S1 - Hbar[:, :, None]", "dev = S1"),
    "routing weight sign flipped": ("scores + lam * np.asarray(route", "scores - lam * np.asarray(route"),
    "routing bias on the query axis": ("dtype=np.float64)[:, :, None, :]", "dtype=np.float64)[:, :, :, None]"),
    "bf16 rounding truncates": ("r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16", "r = (u >> 16) << 16"),
    "dense scale missing": ("z = scale * np.matmul(Q, np.swapaxes(K, -1, -2))",
                            "z = np.matmul(Q, np.swapaxes(K, -1, -2))"),
    "dense max over the query axis": ("z = z - z.max(axis=-1, keepdims=True)",
                                      "z = z - z.max(axis=-2, keepdims=True)"),
    "dense normaliser over queries": ("np.matmul(p, V) / p.sum(axis=-1, keepdims=True)",
                                      "np.matmul(p, V) / p.sum(axis=-2, keepdims=True)[..., :1]"),
    "proxy from the group's first block only": ("proxy = Q[b, h, s:e].sum(axis=0) / (e - s)",
                                                "proxy = qbar[b, h, m * group]"),
    "members not refined to the candidates": ("_top(row, topk, among=cand)", "_top(row, topk)"),
    "group span one token short": ("span = group * block", "span = group * block - 1"),
    "candidates ranked lowest first": ("order = np.lexsort((cols, -vals))", "order = np.lexsort((cols, vals))"),
    "bf16 ties away from even": ("r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16",
                                 "r = ((u + 0x8000) >> 16) << 16"),
}


@pytest.mark.parametrize("label", list(MUTATIONS))
def test_planted_mistake_is_caught(label):
    old, new = MUTATIONS[label]
    src = open(ORACLE_SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    failed = [n for n, (_, ok) in _pins(mod).items() if not ok]
    assert failed, f"no pin caught: {label}"

"""Helpers shared by the GPU parity tests: moving generated inputs to the
device, running the oracle on the same bf16-rounded values, and the error
measures with the tolerances that the outputs must meet."""
from __future__ import annotations

import numpy as np

import oracle
import workloads as W

# Output tolerances: max abs error and L1-relative error sum|o - o*| / sum|o*|.
MAX_ABS = 1e-2
MEAN_REL = 5e-3


def to_device(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_f64(bits: np.ndarray) -> np.ndarray:
    return W.bf16_bits_to_f32(bits).astype(np.float64)


def bf16_to_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def errors(out: np.ndarray, ref: np.ndarray):
    diff = np.abs(out - ref)
    return float(diff.max()), float(diff.sum() / np.abs(ref).sum())


def assert_close(out, ref, what=""):
    mx, rel = errors(out, ref)
    assert mx <= MAX_ABS and rel <= MEAN_REL, f"{what}: max abs {mx:.3e}, mean rel {rel:.3e}"
    return mx, rel


# (label, rows, oracle near-tie rows, GPU rows differing, of which at near-ties), one
# entry per index comparison of the session; printed by the terminal summary hook
NEAR_TIE_LOG = []


def compare_idx(gpu_idx: np.ndarray, ref_idx: np.ndarray, near: np.ndarray, label: str = ""):
    """Rows must match exactly unless the oracle recorded a near-tie there.
    Returns (mismatched rows, of which near-ties, the mismatch mask) and records the
    counts for the session's near-tie report."""
    bad = np.any(gpu_idx != ref_idx, axis=-1)
    NEAR_TIE_LOG.append((label, int(bad.size), int(near.sum()), int(bad.sum()), int((bad & near).sum())))
    return int(bad.sum()), int((bad & near).sum()), bad


def sampled_query_blocks(wl, count: int = 32, seed: int = 0):
    """Query blocks for a sampled oracle check of a large launch: the first and last
    blocks, and blocks spread over the sequence. At b = 64 both query blocks of each
    chosen 128-row tile are taken (the fused kernel computes two query blocks per tile)."""
    rng = np.random.default_rng(seed)
    def spread(n, k):        # 0, n - 1 and k - 2 others
        inner = rng.choice(np.arange(1, n - 1), size=max(0, min(n - 2, k - 2)), replace=False) if n > 2 else []
        return sorted({0, n - 1} | set(int(x) for x in inner))
    if wl.block == 64:
        qbs = [q for t in spread(-(-wl.nB // 2), count // 2) for q in (2 * t, 2 * t + 1) if q < wl.nB]
    else:
        qbs = spread(wl.nB, count)
    return qbs


def oracle_stats(Kf, Vf, wl: W.Workload):
    """kbar, S0 and the order's first-order statistic (per-block S1 at order 1, the
    head's Hbar at order 2, None otherwise)."""
    kbar, S0, S1 = oracle.block_stats(Kf, Vf, wl.block, 1 if wl.order >= 1 else 0)
    if wl.order == oracle.ORDER_HYBRID:
        S1 = oracle.global_first_order(S1)
    return kbar, S0, S1


def check_first_order_stat(gpu_S1, ref_S1, order: int):
    """Per-block S1 (bf16, one rounding) or Hbar (fp32 sum of fp32 terms)."""
    if order == 1:
        g1 = bf16_to_f64(gpu_S1)
        assert np.all(np.abs(g1 - ref_S1) <= 2.0 ** -8 * np.abs(ref_S1) + 1e-3)
    elif order == 2:
        g = gpu_S1.double().cpu().numpy()
        scale = np.abs(ref_S1).max()
        # fp32 terms of magnitude ~|S1_j| summed over the blocks: allow 1e-4 of the largest entry
        assert np.abs(g - ref_S1).max() <= 1e-4 * scale + 1e-5, np.abs(g - ref_S1).max() / scale


def oracle_pipeline(Qf, Kf, Vf, wl: W.Workload, query_blocks=None):
    """Oracle stats -> select -> attention on fp64 copies of the inputs."""
    kbar, S0, S1 = oracle_stats(Kf, Vf, wl)
    idx, near, _ = oracle.select(Qf, kbar, wl.block, wl.topk)
    O = oracle.attention(Qf, Kf, Vf, kbar, S0, S1, idx, wl.block, wl.order, wl.scale,
                         query_blocks=query_blocks)
    return dict(kbar=kbar, S0=S0, S1=S1, idx=idx, near=near, O=O)

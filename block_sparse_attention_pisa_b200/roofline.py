"""Algorithmic work of each kernel (what PISA must do, not the dense work it avoids).

Per-unit figures:

* attention: 4*b*d flops per (query, critical block) -- QK^T and PV --
  plus 4*d per (query, non-critical block) -- x.kbar and alpha*S0 (orders 0,
  1, 2) -- plus, at order 1, 2*d*d per (query, non-critical block) -- S1^T x --
  or, at order 2 (hybrid), 2*d*d once per query -- x Hbar. Keep-or-drop
  (order -1) has the exact term only. Ragged blocks count at their mean size
  N / nB.
* stats: bytes = K and V read (2*N*d*2 per head) + kbar and S0 written
  (2*nB*d*4) + S1 written (nB*d*d*2 at order 1) or Hbar written (d*d*4 at
  order 2); flops = 2*n*d*d per block for K^T V (orders 1 and 2).
* select: bytes = Q read (N*d*2) + kbar read (nB*d*4) + idx written
  (nB*k*4); flops = 2*d per (query block, key block) pooled score; grouped:
  2*d per (proxy, key block) + 2*d per (member block, candidate).
* routing (covariance-aware): bytes = per-block S1 read twice (2*nB*d*d*2:
  once for Hbar, once for the deviations) + Hbar written and read (2*d*d*4)
  + M written (nB*4).
* dense-equivalent attention flops: 4*N*N*d per head.
"""
from __future__ import annotations


def num_blocks(N: int, block: int) -> int:
    return -(-N // block)


def attention_flops(B, H, N, d, block, topk, order) -> float:
    nB = num_blocks(N, block)
    mean_n = N / nB
    rest = nB - topk
    per_q = 4.0 * mean_n * d * topk
    if order >= 0:
        per_q += 4.0 * d * rest
    if order == 1:
        per_q += 2.0 * d * d * rest
    elif order == 2 and rest > 0:
        per_q += 2.0 * d * d
    return float(B * H * N * per_q)


def _first_order_bytes(nB, d, order) -> int:
    return nB * d * d * 2 if order == 1 else (d * d * 4 if order == 2 else 0)


def attention_bytes(B, H, N, d, block, topk, order) -> float:
    """Compulsory HBM traffic of one attention call (each operand once)."""
    nB = num_blocks(N, block)
    qkvo = 4 * N * d * 2
    stats = (2 * nB * d * 4 if order >= 0 else 0) + _first_order_bytes(nB, d, order)
    return float(B * H * (qkvo + stats + nB * topk * 4))


def dense_flops(B, H, N, d) -> float:
    return 4.0 * B * H * N * N * d


def stats_bytes(B, H, N, d, block, order) -> float:
    nB = num_blocks(N, block)
    return float(B * H * (2 * N * d * 2 + 2 * nB * d * 4 + _first_order_bytes(nB, d, order)))


def stats_flops(B, H, N, d, block, order) -> float:
    return float(B * H * 2.0 * N * d * d) if order >= 1 else 0.0


def select_bytes(B, H, N, d, block, topk) -> float:
    nB = num_blocks(N, block)
    return float(B * H * (N * d * 2 + nB * d * 4 + nB * topk * 4))


def routing_bytes(B, H, N, d, block) -> float:
    nB = num_blocks(N, block)
    return float(B * H * (2 * nB * d * d * 2 + 2 * d * d * 4 + nB * 4))


def select_flops(B, H, N, d, block, group: int = 1, cand: int = 0) -> float:
    """Pooled-score flops: 2 d per (query block, key block) for plain selection; with
    grouped proxies 2 d per (proxy, key block) plus 2 d per (member, candidate) (none
    when the candidate list is handed over unchanged)."""
    nB = num_blocks(N, block)
    if group == 1 and cand in (0, nB):
        return float(B * H * 2.0 * nB * nB * d)
    ng = -(-nB // group)
    c = nB if cand == 0 else cand
    return float(B * H * 2.0 * d * (ng * nB + nB * c))


def step_flops(B, H, N, d, block, topk, order) -> float:
    return (attention_flops(B, H, N, d, block, topk, order) + stats_flops(B, H, N, d, block, order)
            + select_flops(B, H, N, d, block))

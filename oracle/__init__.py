"""CPU fp64 oracle for PISA piecewise sparse attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
this package. The product (``block_sparse_attention_pisa_b200``) never imports
it and shares no code with it.

Source: "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
Transformers" (Li, Shao, Zhong, Zhou, Bai, Xiong, Xie, 2026; explainer page at
gist.science, paper 2602.01077), technical summary section 2, Methodology.
The page names the method's pieces but prints only the numerator; the
first-order term used here is the per-block Taylor term
``e^{x.kbar_B} (S0_B + S1_B^T x)`` with ``S1_B = sum_j (k_j - kbar_B) v_j^T``
and denominator ``n_B e^{x.kbar_B}``, which is the expansion of exp(x.k) to
first order around the block's mean key.

Every function works in float64 on whatever values it is given (the tests pass
the same bf16-rounded values that the GPU receives). Parity pins: every
function here is pinned by tests in ``tests/test_oracle_pins.py`` (brute force
on tiny inputs, closed forms, reductions to textbook softmax attention,
convergence rates, and an independent second formulation of the first-order
term).
"""
from .pisa import (  # noqa: F401
    block_bounds,
    block_stats,
    pooled_queries,
    select,
    select_grouped,
    attention,
    dense_attention,
    global_first_order,
    routing_norms,
    round_to_bf16,
    ORDER_DROP,
    ORDER_ZERO,
    ORDER_FIRST,
    ORDER_HYBRID,
)

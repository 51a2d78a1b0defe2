"""Float64 CPU oracle for alpha-entmax attention.

TEST INFRASTRUCTURE ONLY. This package is the slow, obviously-correct
definition that the CUDA path is checked against. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import it. The library in
``differentiable_sparse_attention_b200`` never imports it and has no CPU
fallback; the two share no code.

Citations name the gist.science summary pages of "AdaSplash-2: Faster
Differentiable Sparse Attention" by their language (zh, it, ja, es) and the
section on that page.  ``dash_router`` covers the stage-0/1 router of
DashAttention from the Italian summary of that paper, which the same pages
carry.
"""

from . import dash_router  # noqa: F401
from .entmax_oracle import (  # noqa: F401
    attention_backward,
    attention_forward,
    attention_windowed,
    block_margins,
    entmax,
    entmax_jvp,
    entmax_probs,
    entmax_threshold,
    histogram_threshold,
    pack_block_mask,
    scores,
)

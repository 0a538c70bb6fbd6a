"""fp64 CPU oracle for Loki decode-time sparse attention.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, obviously correct
restatement of what the Loki pages define. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it. The library path (the CUDA kernels behind the C ABI and their Python
binding) never imports, calls or falls back to it, and it shares no code with
that path: its only common dependency is the seeded input generator
(``workloads``), which holds none of the method's arithmetic.

Source pages (cited by title and section in each function):
  * "Loki: Low-Rank Keys for Efficient Sparse Attention", NeurIPS 2024 poster
    page (deep-diver.github.io): TL;DR; "Visual Insights" Figure 1 caption and
    Table 1 caption; "Loki's Computational Cost"; the figure captions under
    "More on figures" and the table captions under "More on tables".
  * the study.space summary page of the same paper (PCA on keys, top-k on
    low-dimensional scores).
  * the briefgpt.xyz abstract page (tokens ranked and selected by attention
    scores computed in a low-dimensional space).

Every function here is pinned by ``tests/test_oracle_*.py`` against something
other than itself (closed forms, hand-worked fixtures under ``tests/golden/``,
brute force on tiny inputs, invariants of the definitions).
"""
from .loki import (  # noqa: F401
    covariance,
    calibrate_pca,
    calibrate_pca_heads,
    explained_variance_rank,
    round_to_dtype,
    rotate_keys,
    project_query,
    lowdim_scores,
    select_topk,
    attend,
    loki_decode_row,
    dense_decode_row,
    loki_decode,
    dense_decode,
    pca_attn_row,
    prerotary_decode_row,
)

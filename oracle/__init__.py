"""CPU oracle for the NABLA hot path -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, obviously-correct NumPy fp64 restatement of what the
NABLA method computes.  It exists to check the CUDA path.  Only the test suite
(``tests/``), ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The product library (``adaptive_block_sparse_b200``)
never imports, links or calls anything here, and nothing here imports the product.

Sources (web pages describing NABLA, arXiv 2507.13546):
  * "NABLA: Neighborhood Adaptive Block-Level Attention" (gist.science, Chinese edition),
    technical summary, section "Methodology" -- the most precise statement of the steps.
  * The lsdiaocha.cn popular-science article on NABLA (traditional Chinese), section 2
    ("NABLA algorithm's core innovation") and section 4 ("technical principles").

Every function cites the passage it follows.  Where the pages are silent the reading
taken is stated in the docstring.  Pins: see ``tests/test_oracle_*.py``; every function
here is pinned by at least one test that does not restate its formula.
"""

from .nabla import (  # noqa: F401
    fractal_permutation,
    reorder,
    inverse_reorder,
    pool_blocks,
    pooled_logits,
    pooled_softmax,
    cdf_keep_row,
    cdf_mask,
    sta_mask,
    nabla_mask,
    pack_mask_bits,
    unpack_mask_bits,
    row_lists,
    col_lists,
    block_sparse_attention,
    block_sparse_attention_rows,
    block_sparse_attention_bwd,
)

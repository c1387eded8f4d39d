"""Plain CPU oracle for RainFusion rf_v2 block-sparse video attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package:
only the tests, the smoke check and the CPU-baseline leg of the benchmark
use it.  It shares no code, table or constant generator with the CUDA
library; the two meet only through the seeded input generator, which holds
none of the method's arithmetic.

Everything is fp64 numpy (bf16 inputs are widened exactly), written for a
reader to check against the pages by eye.  See ``rf_v2.py`` for the
definitions and the citation of each step.
"""

from .rf_v2 import (  # noqa: F401
    BLOCK,
    TILE,
    Geometry,
    geometry,
    is_dense,
    kept_count,
    pool_blocks,
    block_scores,
    topk_mask,
    build_mask,
    key_set,
    attention_rows,
    dense_attention,
    rf_sparse_attention,
    to_bnsd,
    from_bnsd,
)
from . import fp8  # noqa: F401

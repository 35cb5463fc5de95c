"""FP64 CPU oracle for DiT joint attention (RoPE + softmax attention, BF16 and
FP8 paths).

TEST INFRASTRUCTURE ONLY: the parity tests, the package's smoke check and the
benchmark's CPU-baseline leg are the only callers.  It shares no code with the
CUDA library (no common kernels, helpers, tables or constants) and imports
nothing from it; only the seeded input generator feeds both.

Parity pins: every function here is checked in ``tests/test_oracle_*.py``
against closed forms, invariants, special cases and library routines that do
not reuse its own formulas (see each test's docstring).  ``rounding_ambiguous``
is a test helper, not part of the method.
"""
from .joint_attention import (  # noqa: F401
    as_f64, rope_frequencies, rope_angles, rope_rotate, rms_norm, qk_norm_streams, joint_sequence,
    attention_rows, joint_attention, rotated_qkv, attention_on, flops,
)
from .repair import (  # noqa: F401
    repair_count, repair_scores, repair_select, repaired_attention_rows, repaired_attention,
)
from .block_sparse import (  # noqa: F401
    block_means, block_shares, block_select, block_sparse_attention_rows, block_sparse_attention,
)
from .fp8 import (  # noqa: F401
    E4M3_MAX, e4m3_decode, e4m3_encode, block_scales, quantize_blocks,
    dequantize_blocks, rounding_ambiguous,
)

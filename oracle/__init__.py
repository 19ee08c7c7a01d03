"""fp64 CPU oracle for the MoBA causal prefill forward.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the package smoke check and
by the benchmark's CPU-baseline leg, never by the product path.
"""
from .oracle import (  # noqa: F401
    Oracle, bf16_bits, online_softmax_merge, cu_from_lengths, local_block_info,
    static_selection,
)

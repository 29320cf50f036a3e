"""Float64 CPU oracle (test infrastructure only; never on the product path).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package. It shares no code with the CUDA library.
"""
from .attn_jvp_oracle import (  # noqa: F401
    BLOCK_CAUSAL, TEACHER_FORCING, allowed, attn_forward_dense, attn_jvp_dense,
    attn_jvp_rows, count_pairs_bruteforce, mask_matrix, seq_len,
)

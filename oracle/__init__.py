"""CPU oracle (test infrastructure only; see tasq_oracle for what it computes and why)."""
from .tasq_oracle import (  # noqa: F401
    INT8_QMAX,
    bitops,
    block_hadamard_exact,
    block_hadamard_fp32,
    dequant,
    int_gemm,
    lsb_mask,
    masked_linear,
    pad_rows,
    padded_k,
    prologue,
    quantize_per_token,
    sylvester_hadamard,
)

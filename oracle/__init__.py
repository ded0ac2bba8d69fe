"""Plain CPU oracle for the blockwise-FP8 linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference leg may import this package.  The product (the CUDA library under
``blockwise_fp8_linear_fp8bq_b200``) never imports it, and the two share no
code.  See ``fp8bq_oracle.c`` for the definition each function follows and the
page sections it cites.
"""
from .oracle import (  # noqa: F401
    SCALE_FP32,
    SCALE_UE8M0,
    GRAN_ROW,
    GRAN_BLOCK,
    GRAN_ROW32,
    build,
    lib,
    num_threads,
    e4m3_decode,
    e4m3_encode,
    ue8m0_exponent,
    quantize_act,
    gemm_accumulate,
    swiglu,
    rmsnorm,
    quantize_act_t,
    quantize_weight,
    row_scale_ld,
    Operand,
    row_operand,
    block_operand,
    gemm,
)

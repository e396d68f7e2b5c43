"""Plain fp64 CPU oracle for DeltaKV residual KV-cache compression.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
baseline leg of the benchmark may import this package.  The product path (the
CUDA library in ``decode_attention_strided_b200``) never imports it, and the
two share no code.

The arithmetic lives in ``deltakv_oracle.c`` (plain C, double precision), which
restates the method of "DeltaKV: Residual-Based KV Cache Compression via
Long-Range Similarity" (gist.science summary, section 3 "Metodologia":
"Struttura della Compressione", "Processo di Compressione" steps 1-4,
"Ricostruzione").  This module only builds that file with gcc, loads it with
ctypes and passes numpy arrays in and out; it does no arithmetic of the
method itself.
"""
from .oracle import (  # noqa: F401
    ACT_GELU_ERF,
    ACT_GELU_TANH,
    ACT_NONE,
    ROUND_BF16,
    ROUND_F32,
    ROUND_NONE,
    ROUND_Q4,
    act,
    attention,
    build,
    compress,
    compress_rows,
    lib_path,
    mlp,
    quantize_row4,
    reconstruct,
    reconstruct_rows,
    round_to,
    select,
)

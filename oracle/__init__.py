"""CPU oracle for the W4A4 + low-rank linear layer (test infrastructure only).

A plain fp64 C implementation (tq_oracle.c) behind ctypes.  Only tests, the
smoke check and the benchmark's CPU-baseline leg use it; the CUDA library never
does.  Every function follows the definition it cites in tq_oracle.c.
"""
from .oracle import (  # noqa: F401
    hadamard, rotate, quantize_sym, pack_int4, unpack_int4, int_gemm,
    round_bf16, lowrank, epilogue, quantize_act, pack_weight, layer,
    num_threads, set_num_threads, swiglu, quantize_asym, layer_asym, layer_qlr, signs_from_bits,
)

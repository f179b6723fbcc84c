"""B200 (sm_100a) W4A4 + low-rank linear layer.

The compute lives in libtq.so (hand-written CUDA for sm_100a behind the C ABI
of include/tq.h); this package only marshals torch tensors into that ABI.
There is no CPU fallback: importing the binding without the built library
raises.
"""
from .tq import (  # noqa: F401
    TQError, lib_path, tq_status_string, tq_version, tq_pack_weight, tq_quantize_act,
    tq_gemm_workspace_bytes, tq_w4a4_lr_gemm, tq_w4a4_lr_gemm_noalloc, tq_debug_w4a4_gemm_acc,
    tq_query_device_status, Workspace, layer_forward, tq_layer_workspace_bytes, tq_w4a4_lr_layer,
    tq_quantize_act_i8, tq_w4a4_lr_gemm_a8, tq_layer_path, tq_pack_gate_up,
    tq_gate_up_workspace_bytes, tq_w4a4_lr_gate_up, tq_quantize_act_asym_i8, tq_weight_code_sums,
    tq_w4a4_lr_gemm_a8_asym, tq_pack_lowrank_q4, tq_quantize_act_qlr_i8, tq_w4a4_lr_gemm_a8_qlr,
    tq_noalloc_query_status, tq_debug_noalloc_set_status, tq_debug_watchdog,
    tq_debug_w4a4_lr_layer_decode, tq_pack_shared_input, split_shared_output,
    tq_pack_weight_rht, tq_quantize_act_rht, tq_w4a4_lr_layer_rht, tq_gemm_a8_workspace_bytes,
)

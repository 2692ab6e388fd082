"""B200-native routed mixture-of-experts FFN with 2-/4-bit block-quantised experts.

The computation lives in ``libqmoe.so`` (CUDA for sm_100a, C ABI in
``include/qmoe.h``). ``_lib`` binds that ABI under the same names; ``model``
adds packed-layer and layer-stack objects. Nothing here computes on the CPU:
without the built library every entry point raises.
"""
from ._lib import (BF16, DOWN, F32, GATE_UP, Q2, Q4, QmoeError, exported_symbols, lib,  # noqa: F401
                   qmoe_bucket, qmoe_bucket_workspace_bytes, qmoe_ffn_prefill, qmoe_ffn_prefill_timed, qmoe_prefill_workspace_bytes,
                   qmoe_decode_workspace_bytes, qmoe_experts, qmoe_ffn_decode, qmoe_launch_count, qmoe_ngram_gather,
                   qmoe_pack,
                   qmoe_packed_bytes, qmoe_read_status, qmoe_residual_route, qmoe_rmsnorm_residual, qmoe_route,
                   qmoe_route_fixed, qmoe_route_workspace_bytes, qmoe_stack_buffers, qmoe_stack_create, qmoe_stack_decode,
                   qmoe_stack_decode_host, qmoe_stack_desc, qmoe_stack_destroy, qmoe_stack_kernels_per_replay, qmoe_stack_layer_times,
                   qmoe_stack_path,
                   qmoe_stack_workspace_bytes, qmoe_status_string)

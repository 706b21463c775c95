"""Frozen GGUF-quantized base + LoRA layer for NVIDIA B200 (sm_100a).

The kernels live in ``libqlora.so`` (built from ``csrc/`` by ``build.py``) behind the C ABI of
``include/qlora.h``; ``_lib`` binds that ABI with the same names (torch tensors in, argument
marshalling only). ``inputs`` holds the seeded synthetic workloads and the offline GGUF packers.
"""
from ._lib import (  # noqa: F401
    Q2_K, Q4_0, Q4_K, Q5_K, Q6_K, Q8_0, QL_BF16, QL_F32, QloraError, lib,
    gguf_dequant,
    qlora_linear_workspace_bytes, qlora_linear_fwd, qlora_linear_bwd, qlora_linear_fwd_noalloc,
    MoeRoute, qlora_moe_route_workspace_bytes, qlora_moe_route, qlora_moe_saved_bytes, qlora_moe_workspace_bytes,
    qlora_moe_fwd, qlora_moe_bwd,
    qlora_lm_head_ce_workspace_bytes, qlora_lm_head_ce,
    qlora_rmsnorm_fwd, qlora_rmsnorm_bwd,
    Adamw8State, qlora_adamw8_step,
    qlora_device_status, qlora_launch_count, qlora_selftest_wait_timeout, qlora_set_kernel_events,
    qlora_set_rows_fusion, qlora_status_string)

"""The oracle: a plain, slow, fp64 CPU statement of what the layer computes.

TEST INFRASTRUCTURE ONLY. The library never imports, calls or links anything here; only the tests,
the smoke check and the benchmark's CPU-baseline leg do. It shares no code with the CUDA path:
its inputs come from the seeded generators (``quantized_base_lora_tma_b200.inputs``), which hold
none of the method's arithmetic.

Modules
  gguf_blocks   exact decode of Q4_0 / Q8_0 / Q4_K blocks and the fp32 / bf16 roundings
  lora_linear   dense frozen-base + LoRA linear, forward and backward
  moe           routing and the routed SwiGLU expert layer with LoRA, forward and backward

Parity status: every function here is pinned by the ``-m "not gpu"`` tests (hand-packed blocks,
an independent GGUF decoder, closed forms, finite differences, brute-force loops).
"""

"""B200-native (sm_100a) Fast-dLLM block-decoding step.

  block_kv_cache_b200.fdllm  - binding of the C-ABI library libfdllm.so
  block_kv_cache_b200.synth  - seeded synthetic workloads
  block_kv_cache_b200.build  - nvcc build of libfdllm.so (in-tree)
"""

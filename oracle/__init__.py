"""CPU oracle for the Fast-dLLM block-decoding step.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the product path. See fastdllm.py.
"""
from .fastdllm import *  # noqa: F401,F403
from .fastdllm import (attention, dualcache_attention, kv_store,  # noqa: F401
                       confidence_from_logits, lm_logits, lmhead_confidence,
                       select_positions, threshold_unmask, full_forward,
                       full_hidden, block_forward, block_hidden, prefix_forward,
                       prefix_hidden, generate_dualcache, generate_prefixcache, generate_nocache,
                       generate_sequential, apply_rope, rms_norm, silu,
                       tau_as_single, Confidence, DecodeTrace)

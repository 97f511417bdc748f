"""CPU oracle for the Fast-dLLM block-decoding step.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the product path. See fastdllm.py.
"""
from .fastdllm import *  # noqa: F401,F403
from .fastdllm import (attention, dualcache_attention, kv_store,  # noqa: F401
                       confidence_from_logits, lm_logits, lmhead_confidence,
                       select_positions, threshold_unmask, full_forward,
                       block_forward, generate_dualcache, generate_nocache,
                       generate_sequential, apply_rope, rms_norm, silu,
                       tau_as_single, Confidence, DecodeTrace)

"""fp64 CPU oracle for the sink + rolling-window KV path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package; the product path never does.
"""
from .sdv2_oracle import *  # noqa: F401,F403
from .sdv2_oracle import (CacheConfig, MotionConfig, MotionState, OracleCache,  # noqa: F401
                          attention_reference, bf16_decode, bf16_encode, bf16_round,
                          chunk_attention, chunk_queries_rotated, cosine, kv_append,
                          motion_noise_rate, rope_axis_cos_sin, rope_pair_split, rope_phase,
                          rope_rotate, rope_token_cos_sin, sink_refresh, slot_frames,
                          slot_of_frame, valid_keys, valid_slot_counts)

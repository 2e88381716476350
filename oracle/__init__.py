"""CPU float64 oracle for exact blockwise (ring) attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: it is used by ``tests/``, by ``__graft_entry__.smoke()``
and by the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.  It
shares no code with the CUDA library (no kernels, headers, helpers or
constants); the only module both sides use is ``workloads`` (seeded random
inputs, no attention arithmetic).

Sources ("the pages"):
  [RA]  "Ring Attention: the secret of million-token context"
        (Ring Attention：百万 Token 上下文的秘密, guijiagi.com):
        §2.1 chunking, §2.2 ring schedule figure, §2.3 correctness equation,
        §3.1 Flash Ring Attention two-level loop.
  [BT]  "Billion-token context window engineering" (blog.hotdry.top),
        "core challenge" paragraph: Attention(Q,K,V) = softmax(QK^T/sqrt(d))V.
  [LC]  "From hundreds of milliseconds to a million tokens"
        (从百毫秒到百万Token, pwwt.cn): attention definition, and system layer 4
        "attention fusion layer" (global softmax normalisation of local outputs).
  [CI]  "RingAttention inference: using cache_idx" (RingAttention推理优化：
        cache_idx参数使用, ldbm.cn): "how cache_idx works" (query chunk start
        from cache_idx), basic inference configuration (causal_block_size=1,
        float32_logits), distributed configuration (ppermute to (i+1) mod n).

Parity status: every public function here is pinned by tests under
``tests/test_oracle_*.py`` against things other than itself (a library
routine, brute force, closed forms, invariants, the pages' printed schedule).
"""
from .attention import (
    attention_bwd_ref,
    attention_fp8kv_ref,
    attention_ref,
    attention_window_anchor_ref,
    block_step_bwd_ref,
    block_step_ref,
    decode_e4m3,
    finalize_ref,
    init_state,
    lse_merge_ref,
    ring_bwd_ref,
    ring_ref,
    ring_visit_chunk,
    query_home_chunk,
    window_anchor_visible,
)

__all__ = [
    "attention_bwd_ref",
    "attention_fp8kv_ref",
    "attention_ref",
    "attention_window_anchor_ref",
    "block_step_bwd_ref",
    "block_step_ref",
    "decode_e4m3",
    "finalize_ref",
    "init_state",
    "lse_merge_ref",
    "ring_bwd_ref",
    "ring_ref",
    "ring_visit_chunk",
    "query_home_chunk",
    "window_anchor_visible",
]

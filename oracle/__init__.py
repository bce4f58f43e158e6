"""CPU oracle for attention over a paged KV cache -- TEST INFRASTRUCTURE ONLY.

This package is the slow, obviously correct statement of what the CUDA path
computes.  It exists so that tests, the smoke check and the benchmark's CPU
baseline leg have something independent to compare against.  Nothing in the
product path (the C-ABI library, its Python binding) imports it, and it
imports nothing from the product package: the two share no code.

Every floating-point computation here is float64.  bf16/fp32 inputs are
up-cast exactly before any arithmetic.

Sources (page title, section):
  * "AI Infra入门干货总结：大模型是如何高效推理的" (enzochen.online clipping of
    the Tencent article), section "Paged Attention": cache layout
    [num_blocks, block_size, num_kv_heads, head_dim], the block_table, the
    slot_mapping formula and its worked example (block_size 16, table
    [5, 8, 12], position 25 -> slot 137).
  * same article, section "Attention (FlashAttention, Scaled Dot-Product
    Attention)": softmax(Q K^T / sqrt(d) + M) V, the GQA index map
    kv_head = q_head // (num_heads // num_kv_heads), the causal mask (future
    positions -inf), the online softmax (running max, running sum, rescale),
    and the unified varlen call that reads every K/V through the block table.
  * same article, section "总结": Flash-Decoding splits the KV axis and
    re-normalises the pieces with log-sum-exp.
  * ursb.me Field Note "llm-inference-life", blurb: running max m, running
    denominator l and the exp(m_old - m_new) correction factor; every pair of
    Q/K dimensions rotated in the complex plane by m*theta (rotary position
    embedding, oracle/rope.py).
  * "第三部分 · 推理系统与基础设施" (llm-learning-path part 3), chapter map,
    3.3: block tables with copy-on-write (oracle/blocks.py); 3.2 / 3.6: KV
    quantisation, FP8 formats (oracle/fp8.py).
  * "从零构建LLM 推理引擎" (llminference.xinbetween.com), card "量化": fewer
    bits per KV entry, fewer bytes per decoded token (oracle/fp8.py).
  * "AI Infra入门干货总结", sections "Reshape & Cache" (Q/K rotated by the
    position's rotation, cos_sin_cache [max_position, rotary_dim], then the
    scatter into the pools) and "附1：模型配置参数" (rope_theta 500000).

Pins: every function here is checked by tests/test_oracle.py against facts
fixed by the pages or by mathematics (the worked slot example, closed forms,
brute force, a library attention routine, invariants).  No function is
"parity unpinned".
"""

from .attention import (  # noqa: F401
    slot_of,
    slot_mapping,
    cache_write,
    gather,
    attend_two_pass,
    attend_online,
    attend_partial,
    merge_partials,
    attend_split,
    paged_decode,
    paged_mixed_step,
    kv_cache_bytes,
    ERR_SLOT_OOB,
    ERR_BLOCK_OOB,
    ERR_SEQ_TOO_LONG,
    ERR_QUERY_TOO_LONG,
)
from .brute import brute_attention  # noqa: F401
from .blocks import (  # noqa: F401
    ERR_POS_OOB_TABLE,
    copy_blocks,
    slot_mapping_positions,
)
from .fp8 import (  # noqa: F401
    E4M3_MAX,
    dequantize,
    e4m3_decode,
    e4m3_encode,
    quantize,
)
from .rope import (  # noqa: F401
    ERR_POS_OOB,
    cos_sin_table,
    inv_freq,
    pair_index,
    rope_cache_write,
    rotate,
)

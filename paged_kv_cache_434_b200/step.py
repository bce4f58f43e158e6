"""One layer's attention step over the paged cache: the three library calls in
the order the vLLM v1 walkthrough gives them ("AI Infra入门干货总结：大模型是如何
高效推理的", "Reshape & Cache" then "Attention"): compute the new tokens'
slots, scatter their K/V into the pools, then attend through the block tables.
"""

from __future__ import annotations

import torch

from . import binding


def step(q, k_new, v_new, k_cache, v_cache, block_tables, query_start_loc, seq_lens,
         scale: float, *, decode_only: bool = False, out=None, out_dtype=torch.float32,
         slots=None, workspace=None, err=None, kv_scales=None):
    """Run slot_mapping -> cache_write -> decode / mixed_step on the current
    stream: a decode step in one call (the write rides in the planner's
    launch), a mixed step as the fused slot/cache write then the attention.

    q: [T, Hq, D]; k_new, v_new: [T, Hkv, D]; query_start_loc: [B+1] int32;
    seq_lens: [B] int32 (lengths after this step).  float8_e4m3fn pools take
    kv_scales=(k_scale, v_scale) and bf16 q / k_new / v_new.  With decode_only=True every
    request has exactly one new token (T == B) and pa_decode is used.
    Returns out [T, Hq, D].
    """
    if decode_only:  # token b belongs to request b: no query offsets needed
        return binding.decode_step(q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens,
                                   scale, out=out, out_dtype=out_dtype, slots=slots,
                                   workspace=workspace, err=err, kv_scales=kv_scales)[0]
    binding.slot_mapping_cache_write(k_new, v_new, k_cache, v_cache, block_tables,
                                     query_start_loc, seq_lens, slots=slots, err=err,
                                     kv_scales=kv_scales)
    return binding.mixed_step(q, k_cache, v_cache, block_tables, query_start_loc, seq_lens, scale,
                              out=out, out_dtype=out_dtype, workspace=workspace, err=err,
                              kv_scales=kv_scales)

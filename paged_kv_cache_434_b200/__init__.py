"""paged_kv_cache_434_b200 -- attention over a paged KV cache on B200 (sm_100a).

The compute lives in libpa_b200.so (C ABI in include/pa.h); this package is
its Python binding plus a seeded workload generator:

  slot_mapping   slot of every new token from the block tables
  cache_write    reshape_and_cache into [num_blocks, block_size, Hkv, D] pools
  rope_cache_write  rotary embedding of Q/K fused with the cache write
  rope_cos_sin_cache  the [max_position, rotary_dim] cos/sin table
  copy_blocks    copy-on-write block copies in both pools
  slot_mapping_positions  slots from explicit (request, position) pairs
  decode         GQA decode attention, online softmax, split-KV + LSE merge
  decode_no_alloc  decode through the library's own static scratch
  decode_step    a decode step's cache write and attention in one call
  mixed_step     causal varlen attention of a chunked-prefill + decode step
  step           slot_mapping -> cache_write -> attention, the per-layer path
"""

from .binding import (  # noqa: F401
    ERRBIT_BLOCK_OOB,
    ERRBIT_QUERY_TOO_LONG,
    ERRBIT_SEQ_TOO_LONG,
    ERRBIT_SLOT_OOB,
    ERRBIT_POS_OOB,
    ERRBIT_Q_RANGE,
    ERRBIT_TIMEOUT,
    PagedAttentionError,
    cache_write,
    copy_blocks,
    decode,
    decode_no_alloc,
    decode_step,
    decode_workspace_size,
    kernel_times,
    kernel_timing,
    library_path,
    mixed_step,
    mixed_step_workspace_size,
    new_error_word,
    read_error,
    rope_cache_write,
    rope_cos_sin_cache,
    slot_mapping,
    slot_mapping_cache_write,
    slot_mapping_positions,
    version,
)
from .step import step  # noqa: F401

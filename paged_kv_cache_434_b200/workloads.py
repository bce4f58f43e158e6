"""Seeded synthetic workloads for paged-KV attention.

This module only draws inputs: sequence lengths, the order in which a block
allocator hands out physical block ids, and N(0, 1) values for Q, the new
tokens' K/V and the pre-filled history in the cache pools.  It holds none of
the attention arithmetic (no slot computation, no softmax); the CUDA library
and the CPU oracle both consume what it produces.

Geometries and batch mixes follow the workloads the pages talk about: the
Llama-3-8B layer (32 query heads, 8 KV heads, head_dim 128, "附1：模型配置参数"),
block_size 16 (the vLLM default named in "Paged Attention"), decode batches,
long contexts that need split-KV, a chunked-prefill continuous-batching step,
and a batch sharing a cached prefix.

Random streams:
  * lengths / orders: numpy PCG64 seeded with (seed, stream tag);
  * values: float32 N(0, 1), then rounded to the compute dtype (RNE for bf16).
    Small workloads draw on the host with numpy PCG64; large pools are drawn
    on the device with a seeded torch CUDA generator, in slices, so that tens
    of GB never pass through host memory.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

TAG_LENS, TAG_PERM, TAG_VALUES, TAG_ORDER = 1, 2, 3, 4
VALUE_TAGS = {"q": 11, "k_new": 12, "v_new": 13, "k_cache": 14, "v_cache": 15}


@dataclasses.dataclass
class Workload:
    """Shape and index structure of one flattened step (no tensor values)."""

    name: str
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str                     # "f32" or "bf16"
    seq_lens: np.ndarray           # int32 [B]   KV length after this step
    query_lens: np.ndarray         # int32 [B]   new tokens this step
    block_tables: np.ndarray       # int32 [B, W] physical ids, -1 past the end
    num_blocks: int                # pool size (physical blocks)
    scale: float
    seed: int
    shared_prefix_blocks: int = 0  # leading table entries common to all rows
    kv_dtype: str = ""             # "fp8": e4m3 pools (q / new K/V stay bf16)
    kv_scale: float = 1.0          # fp8 pools: an entry stands for code * kv_scale

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def query_start_loc(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.query_lens)]).astype(np.int32)

    @property
    def num_tokens(self) -> int:
        return int(self.query_lens.sum())

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def elt_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def pool_elt_bytes(self) -> int:
        return 1 if self.kv_dtype == "fp8" else self.elt_bytes

    @property
    def kv_scales(self):
        return (self.kv_scale, self.kv_scale) if self.kv_dtype == "fp8" else None

    @property
    def is_decode(self) -> bool:
        return bool(np.all(self.query_lens == 1))


def _rng(seed: int, tag: int) -> np.random.Generator:
    return np.random.default_rng([seed, tag])


def _blocks_for(length: int, block_size: int) -> int:
    return (int(length) + block_size - 1) // block_size


def _tables_from_order(lens, block_size, order, width=None, start=0):
    """Hand out physical ids from `order` to each request, in request order."""
    need = [_blocks_for(L, block_size) for L in lens]
    width = max(max(need), 1) if width is None else width
    tables = np.full((len(lens), width), -1, dtype=np.int32)
    cursor = start
    for b, n in enumerate(need):
        tables[b, :n] = order[cursor:cursor + n]
        cursor += n
    return tables, cursor


def custom(name, seq_lens, query_lens, num_heads, num_kv_heads, head_dim, block_size,
           dtype, seed=0, extra_blocks=0, scale=None, table_width=None):
    """Generic workload: pool = blocks needed (+ extra), ids randomly permuted."""
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    query_lens = np.asarray(query_lens, dtype=np.int32)
    need = sum(_blocks_for(L, block_size) for L in seq_lens)
    num_blocks = max(need + extra_blocks, 1)
    order = _rng(seed, TAG_PERM).permutation(num_blocks).astype(np.int32)
    tables, _ = _tables_from_order(seq_lens, block_size, order, width=table_width)
    return Workload(name, num_heads, num_kv_heads, head_dim, block_size, dtype,
                    seq_lens, query_lens, tables, num_blocks,
                    scale if scale is not None else 1.0 / math.sqrt(head_dim), seed)


def tiny_decode(seed: int = 0) -> Workload:
    """3 sequences of 25, 9 and 40 tokens; 8 query / 2 KV heads, head_dim 64,
    fp32, block_size 16, a 16-block pool with ids from a seeded permutation."""
    lens = np.array([25, 9, 40], dtype=np.int32)
    order = _rng(seed, TAG_PERM).permutation(16).astype(np.int32)
    tables, _ = _tables_from_order(lens, 16, order)
    return Workload("tiny_decode_fp32", 8, 2, 64, 16, "f32", lens,
                    np.ones(3, dtype=np.int32), tables, 16, 1.0 / math.sqrt(64), seed)


def llama8b_decode(seed: int = 0, num_seqs: int = 64, min_len: int = 512,
                   max_len: int = 8192) -> Workload:
    """Llama-3-8B layer decode: 64 sequences, lengths uniform in [512, 8192]."""
    lens = _rng(seed, TAG_LENS).integers(min_len, max_len + 1, size=num_seqs).astype(np.int32)
    w = custom("llama3_8b_decode_bf16", lens, np.ones(num_seqs, np.int32), 32, 8, 128, 16,
               "bf16", seed, table_width=_blocks_for(max_len, 16))
    return w


def long_context_decode(seed: int = 0) -> Workload:
    """4 sequences of 32K, 64K, 96K and 128K tokens at the Llama-3-8B geometry."""
    lens = np.array([32768, 65536, 98304, 131072], dtype=np.int32)
    return custom("long_context_split_kv_bf16", lens, np.ones(4, np.int32), 32, 8, 128, 16,
                  "bf16", seed)


def mixed_step(seed: int = 0, shuffle: bool = False, num_decodes: int = 4096,
               chunk: int = 2048, prefix: int = 4096) -> Workload:
    """Continuous-batching step with a token budget of 8192.

    Request 0: a 2048-token chunk continuing a 4096-token cached prefix
    (seq_len 6144, query_len 2048).  Request 1: a fresh 2048-token prompt
    chunk.  Then 4096 decodes with one query each and context uniform in
    [1024, 4096].  With shuffle=True the request order is permuted.
    """
    dec_lens = _rng(seed, TAG_LENS).integers(1024, 4097, size=num_decodes)
    lens = np.concatenate([[prefix + chunk, chunk], dec_lens]).astype(np.int32)
    qlens = np.concatenate([[chunk, chunk], np.ones(num_decodes)]).astype(np.int32)
    if shuffle:
        perm = _rng(seed, TAG_ORDER).permutation(len(lens))
        lens, qlens = lens[perm], qlens[perm]
    return custom("mixed_chunked_prefill_bf16", lens, qlens, 32, 8, 128, 16, "bf16", seed)


def shared_prefix_decode(seed: int = 0, num_seqs: int = 128, prefix_tokens: int = 4096,
                         block_size: int = 32) -> Workload:
    """70B-style decode (64 query / 8 KV heads) whose block tables all start
    with the same 128 physical blocks (a 4096-token shared prefix), followed
    by unique suffixes of 256..1024 tokens in randomly permuted blocks."""
    suffix = _rng(seed, TAG_LENS).integers(256, 1025, size=num_seqs)
    lens = (prefix_tokens + suffix).astype(np.int32)
    pblocks = prefix_tokens // block_size
    sblocks = [_blocks_for(s, block_size) for s in suffix]
    num_blocks = pblocks + sum(sblocks)
    order = _rng(seed, TAG_PERM).permutation(num_blocks).astype(np.int32)
    width = pblocks + max(sblocks)
    tables = np.full((num_seqs, width), -1, dtype=np.int32)
    tables[:, :pblocks] = order[:pblocks]
    cursor = pblocks
    for b, n in enumerate(sblocks):
        tables[b, pblocks:pblocks + n] = order[cursor:cursor + n]
        cursor += n
    return Workload("shared_prefix_70b_decode_bf16", 64, 8, 128, block_size, "bf16", lens,
                    np.ones(num_seqs, np.int32), tables, num_blocks, 1.0 / math.sqrt(128),
                    seed, shared_prefix_blocks=pblocks)


def mixed_step_prefill_only(seed: int = 0, chunk: int = 2048, prefix: int = 4096) -> Workload:
    """Only the two chunked-prefill requests of mixed_step(): a 2048-token
    chunk after a 4096-token cached prefix and a fresh 2048-token prompt."""
    lens = np.array([prefix + chunk, chunk], dtype=np.int32)
    qlens = np.array([chunk, chunk], dtype=np.int32)
    return custom("mixed_prefill_chunks_bf16", lens, qlens, 32, 8, 128, 16, "bf16", seed)


# --------------------------------------------------------------------------
# Tensor values
# --------------------------------------------------------------------------

def _torch_dtype(dtype: str):
    import torch
    return torch.float32 if dtype == "f32" else torch.bfloat16


def _host_normal(seed: int, tag: int, shape, dtype: str):
    import torch
    x = _rng(seed, TAG_VALUES * 1000 + tag).standard_normal(size=int(np.prod(shape)),
                                                            dtype=np.float32)
    return torch.from_numpy(x).reshape(shape).to(_torch_dtype(dtype))


def _device_normal_(out, seed: int, tag: int, slice_elems: int = 1 << 28):
    """Fill a CUDA tensor with N(0,1) drawn as float32 and rounded to its dtype."""
    import torch
    gen = torch.Generator(device=out.device)
    gen.manual_seed((seed * 1_000_003 + tag) & 0x7FFFFFFFFFFFFFFF)
    flat = out.view(-1)
    for lo in range(0, flat.numel(), slice_elems):
        hi = min(flat.numel(), lo + slice_elems)
        tmp = torch.randn(hi - lo, generator=gen, device=out.device, dtype=torch.float32)
        flat[lo:hi].copy_(tmp)
        del tmp
    return out


def make_tensors(w: Workload, device="cpu", where: str = "auto"):
    """Draw q [T, Hq, D], k_new / v_new [T, Hkv, D] and the two pools
    [num_blocks, block_size, Hkv, D] for workload `w`.

    where="host" draws everything with numpy on the CPU (and copies to
    `device`); where="device" draws on the CUDA device; "auto" picks the host
    for pools below 2**26 elements.
    """
    import torch
    T, Hq, Hkv, D = w.num_tokens, w.num_heads, w.num_kv_heads, w.head_dim
    pool_shape = (w.num_blocks, w.block_size, Hkv, D)
    shapes = {"q": (T, Hq, D), "k_new": (T, Hkv, D), "v_new": (T, Hkv, D),
              "k_cache": pool_shape, "v_cache": pool_shape}
    if where == "auto":
        where = "host" if (np.prod(pool_shape) < (1 << 26) or str(device) == "cpu") else "device"
    out = {}
    for name, shape in shapes.items():
        if where == "host":
            out[name] = _host_normal(w.seed, VALUE_TAGS[name], shape, w.dtype).to(device)
        else:
            t = torch.empty(shape, dtype=_torch_dtype(w.dtype), device=device)
            out[name] = _device_normal_(t, w.seed, VALUE_TAGS[name])
        if w.kv_dtype == "fp8" and name in ("k_cache", "v_cache"):
            # the same draws, stored as e4m3 codes by torch's own conversion
            # (inputs for both sides; the oracle decodes the codes itself)
            x = torch.clamp(out[name].float() / w.kv_scale, -448.0, 448.0)
            out[name] = x.to(torch.float8_e4m3fn)
    return out


def llama8b_decode_fp8(seed: int = 0) -> Workload:
    """llama8b_decode over e4m3 pools (per-pool scale 1/56)."""
    return with_fp8_cache(llama8b_decode(seed))


def long_context_decode_fp8(seed: int = 0) -> Workload:
    """long_context_decode over e4m3 pools (per-pool scale 1/56)."""
    return with_fp8_cache(long_context_decode(seed))


def with_fp8_cache(w: Workload, scale: float = 1.0 / 56.0) -> Workload:
    """The same workload over e4m3 pools (N(0,1) entries over 1/56: |x| <= 8
    stays below the format's 448)."""
    import dataclasses
    return dataclasses.replace(w, name=w.name + "_fp8kv", dtype="bf16", kv_dtype="fp8",
                               kv_scale=scale)


def index_tensors(w: Workload, device="cpu"):
    """block_tables, seq_lens, query_start_loc as int32 torch tensors."""
    import torch
    return {
        "block_tables": torch.from_numpy(np.ascontiguousarray(w.block_tables)).to(device),
        "seq_lens": torch.from_numpy(np.ascontiguousarray(w.seq_lens)).to(device),
        "query_start_loc": torch.from_numpy(w.query_start_loc).to(device),
    }


def kv_bytes_touched(w: Workload, unique: bool = True) -> int:
    """Algorithmic K+V bytes one pass of attention must read: valid tokens only;
    with unique=True a physical block shared by several tables counts once."""
    row = 2 * w.num_kv_heads * w.head_dim * w.pool_elt_bytes
    if not unique:
        return int(w.seq_lens.astype(np.int64).sum()) * row
    seen = {}
    for b in range(w.num_seqs):
        L = int(w.seq_lens[b])
        for j in range(_blocks_for(L, w.block_size)):
            pid = int(w.block_tables[b, j])
            valid = min(w.block_size, L - j * w.block_size)
            seen[pid] = max(seen.get(pid, 0), valid)
    return sum(seen.values()) * row

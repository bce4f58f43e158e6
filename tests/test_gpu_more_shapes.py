"""Shapes the library accepts beyond the parity suites, against the fp64 oracle:

  * block sizes 64, 128 and 256 (beside 8, 16 and 32) on every kernel path:
    fp32 generic kernel, bf16 mma.sync partitions and tensor-core prefill
    tiles, e4m3 pools, the shared-prefix cascade.  A 16-key stage then
    covers part of one block, and a request's last block is mostly empty;
  * one KV head (MQA) and an odd number of KV heads, where each decode work
    item carries a single KV head (the one-head variant of the mma.sync
    kernel) and the tensor-core tiles take all query heads of the one group.

The `late` mark runs this file after the parity suites.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import workloads as W
from _util import assert_close, bits, f64, fp8_codes, oracle_full, oracle_full_fp8

pytestmark = [pytest.mark.gpu, pytest.mark.late(2)]

BLOCK_SIZES = [64, 128, 256]


def _run_and_check(w, dev):
    host = W.make_tensors(w, "cpu", where="host")
    t = {k: v.to(dev) for k, v in host.items()}
    idx = W.index_tensors(w, dev)
    err = P.new_error_word(dev)
    slots = torch.empty(w.num_tokens, dtype=torch.int64, device=dev)
    out = P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
                 idx["query_start_loc"], idx["seq_lens"], w.scale, decode_only=w.is_decode,
                 slots=slots, err=err, kv_scales=w.kv_scales)
    torch.cuda.synchronize()
    assert P.read_error(err) == 0
    if w.kv_dtype == "fp8":
        ref_slots, kb, vb, ref, ref_err, valid = oracle_full_fp8(w, host)
        assert np.array_equal(fp8_codes(t["k_cache"]), kb)
        assert np.array_equal(fp8_codes(t["v_cache"]), vb)
    else:
        ref_slots, kb, vb, ref, ref_err, valid = oracle_full(w, host)
        assert np.array_equal(bits(t["k_cache"]), kb) and np.array_equal(bits(t["v_cache"]), vb)
    assert ref_err == set()
    assert np.array_equal(slots.cpu().numpy(), ref_slots)
    assert_close(f64(out)[valid], ref[valid], "f32" if w.dtype == "f32" else "bf16", w.name)


def _lens(bs, rng):
    # 1 key, a partial first block, exactly one block, one key more, several blocks
    return [1, bs // 2 + 3, bs, bs + 1, 3 * bs + 17] + rng.integers(1, 1500, 3).tolist()


@pytest.mark.parametrize("bs", BLOCK_SIZES)
@pytest.mark.parametrize("dtype,hq,hkv,d", [("f32", 8, 2, 64), ("bf16", 32, 8, 128),
                                            ("bf16", 8, 2, 64)])
def test_decode_large_blocks(cuda_device, bs, dtype, hq, hkv, d):
    rng = np.random.default_rng([bs, hq, d])
    lens = _lens(bs, rng)
    w = W.custom(f"decode_bs{bs}_{dtype}_{d}", lens, [1] * len(lens), hq, hkv, d, bs, dtype,
                 seed=bs + d, extra_blocks=2)
    _run_and_check(w, cuda_device)


@pytest.mark.parametrize("bs", BLOCK_SIZES)
@pytest.mark.parametrize("dtype,hq,hkv,d", [("f32", 8, 2, 64), ("bf16", 32, 8, 128),
                                            ("bf16", 16, 2, 64)])
def test_mixed_step_large_blocks(cuda_device, bs, dtype, hq, hkv, d):
    # a chunk after a cached prefix, a fresh prompt, decodes
    lens = [bs + 200, 130, 1, 2 * bs + 5, 700]
    qlens = [150, 130, 1, 1, 1]
    w = W.custom(f"mixed_bs{bs}_{dtype}_{d}", lens, qlens, hq, hkv, d, bs, dtype,
                 seed=bs + d + 1)
    _run_and_check(w, cuda_device)


@pytest.mark.parametrize("bs", BLOCK_SIZES)
def test_fp8_decode_large_blocks(cuda_device, bs):
    rng = np.random.default_rng([bs, 8])
    lens = _lens(bs, rng)
    w = W.with_fp8_cache(W.custom(f"fp8_bs{bs}", lens, [1] * len(lens), 32, 8, 128, bs, "bf16",
                                  seed=bs + 3))
    _run_and_check(w, cuda_device)


@pytest.mark.parametrize("bs", BLOCK_SIZES)
def test_shared_prefix_large_blocks(cuda_device, bs):
    # 24 requests whose tables start with the same 1024 tokens of blocks
    w = W.shared_prefix_decode(bs, num_seqs=24, prefix_tokens=1024, block_size=bs)
    _run_and_check(w, cuda_device)


# Block size 16 takes one [dims x 16 keys] box per head and half; block size 8
# takes two [dims x 8 keys] boxes per head and half (a stage spans two blocks).
@pytest.mark.parametrize("bs", [16, 8])
@pytest.mark.parametrize("dtype,hq,hkv,d", [("bf16", 8, 1, 128), ("bf16", 16, 1, 64),
                                            ("bf16", 12, 3, 128), ("bf16", 5, 5, 64),
                                            ("f32", 8, 1, 64)])
def test_decode_single_kv_head_per_item(cuda_device, bs, dtype, hq, hkv, d):
    rng = np.random.default_rng([hq, hkv, d, bs])
    lens = [1, 7, 8, 9, 15, 16, 17, 700, 2500] + rng.integers(1, 1200, 3).tolist()
    w = W.custom(f"decode_mqa_{hq}_{hkv}_{d}_{dtype}_bs{bs}", lens, [1] * len(lens), hq, hkv, d,
                 bs, dtype, seed=hq * 7 + hkv + d + bs, extra_blocks=2)
    _run_and_check(w, cuda_device)


@pytest.mark.parametrize("bs", [16, 8])
@pytest.mark.parametrize("hq,hkv,d", [(8, 1, 128), (16, 1, 64), (12, 3, 128)])
def test_mixed_step_single_kv_head_per_item(cuda_device, bs, hq, hkv, d):
    lens = [400, 130, 1, 37, 900, 9]
    qlens = [150, 130, 1, 1, 1, 1]
    w = W.custom(f"mixed_mqa_{hq}_{hkv}_{d}_bs{bs}", lens, qlens, hq, hkv, d, bs, "bf16",
                 seed=hq * 7 + hkv + d + bs + 1)
    _run_and_check(w, cuda_device)


@pytest.mark.parametrize("hq,hkv", [(8, 1), (12, 3), (16, 4)])
def test_fp8_decode_head_groups(cuda_device, hq, hkv):
    # e4m3 decode with one and with four KV heads per work item
    lens = [1, 16, 17, 900, 2500]
    w = W.with_fp8_cache(W.custom(f"fp8_heads_{hq}_{hkv}", lens, [1] * len(lens), hq, hkv, 128,
                                  16, "bf16", seed=77 + hkv))
    _run_and_check(w, cuda_device)


def test_fp8_query_beyond_f16_range_sets_its_error_bit(cuda_device):
    """Over e4m3 pools the tensor-core decode path takes queries as f16: a
    query entry beyond +-65504 sets PA_ERRBIT_Q_RANGE.  The requests whose
    queries are in range are still exact."""
    dev = cuda_device
    w = W.with_fp8_cache(W.custom("fp8_q_range", [40, 300, 77], [1, 1, 1], 8, 2, 128, 16, "bf16",
                                  seed=91))
    host = W.make_tensors(w, "cpu", where="host")
    host["q"][1, 3, 5] = 1.0e6                       # request 1 only (bf16 holds ~1e6)
    t = {k: v.to(dev) for k, v in host.items()}
    idx = W.index_tensors(w, dev)
    err = P.new_error_word(dev)
    out = P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
                 idx["query_start_loc"], idx["seq_lens"], w.scale, decode_only=True, err=err,
                 kv_scales=w.kv_scales)
    torch.cuda.synchronize()
    assert P.read_error(err) == P.ERRBIT_Q_RANGE
    _, _, _, ref, _, _ = oracle_full_fp8(w, host)
    keep = [0, 2]
    assert_close(f64(out)[keep], ref[keep], "bf16", w.name)

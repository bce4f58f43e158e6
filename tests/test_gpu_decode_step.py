"""pa_decode_step: a decode step's slot mapping, cache write and attention in
one call, the write done by the CTAs beside the work planner.  It must give
what pa_slot_mapping_cache_write then pa_decode give -- the same slots, pools,
outputs and error bits, bit for bit -- and so match the oracle's slot function,
cache write ("AI Infra入门干货总结：大模型是如何高效推理的", sections "Paged
Attention" and "Reshape & Cache") and decode attention ("Attention
(FlashAttention, Scaled Dot-Product Attention)")."""

import numpy as np
import pytest
import torch

import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import workloads as W

from _util import assert_close, bits, f64, fp8_codes, oracle_full

pytestmark = pytest.mark.gpu


def _pool(x):
    return fp8_codes(x) if x.dtype == torch.float8_e4m3fn else bits(x)


def _copies(host, dev):
    return {k: v.to(dev) for k, v in host.items()}


def _two_calls(w, t, idx, err, out_dtype):
    slots = P.slot_mapping_cache_write(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
                                       idx["block_tables"], None, idx["seq_lens"], err=err,
                                       kv_scales=w.kv_scales)
    out = P.decode(t["q"], t["k_cache"], t["v_cache"], idx["block_tables"], idx["seq_lens"],
                   w.scale, out_dtype=out_dtype, err=err, kv_scales=w.kv_scales)
    return out, slots


def _one_call(w, t, idx, err, out_dtype):
    return P.decode_step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
                         idx["block_tables"], idx["seq_lens"], w.scale, out_dtype=out_dtype,
                         err=err, kv_scales=w.kv_scales)


def _compare(w, dev, out_dtype=torch.float32, idx=None, host=None):
    host = host or W.make_tensors(w, "cpu", where="host")
    idx = idx or W.index_tensors(w, dev)
    a, b = _copies(host, dev), _copies(host, dev)
    ea, eb = P.new_error_word(dev), P.new_error_word(dev)
    out_a, slots_a = _two_calls(w, a, idx, ea, out_dtype)
    out_b, slots_b = _one_call(w, b, idx, eb, out_dtype)
    torch.cuda.synchronize()
    bits_b = P.read_error(eb)
    assert bits_b == P.read_error(ea)
    assert torch.equal(slots_a, slots_b)
    for name in ("k_cache", "v_cache"):
        assert np.array_equal(_pool(a[name]), _pool(b[name])), name
    # rows an error leaves unwritten hold whatever torch.empty gave: compare
    # the rows both calls wrote
    rows = torch.ones(out_a.shape[0], dtype=torch.bool, device=dev) if bits_b == 0 else \
        (slots_b >= 0) & (idx["seq_lens"] > 0)
    assert np.array_equal(bits(out_a[rows]), bits(out_b[rows]))
    return host, b, out_b, slots_b, bits_b


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_small_batches(cuda_device, dtype, bs):
    lens = [1, bs, bs + 1, 300, 1000, 77]
    w = W.custom(f"dstep_{dtype}_{bs}", lens, [1] * len(lens), 8, 2, 64, bs, dtype, seed=bs)
    _compare(w, cuda_device)


def test_against_the_oracle(cuda_device):
    """Slots, pools and attention of the one call against the float64 oracle."""
    lens = [5, 16, 17, 129, 700, 2048, 33]
    w = W.custom("dstep_oracle", lens, [1] * len(lens), 32, 8, 128, 16, "bf16", seed=3)
    host, b, out, slots, errbits = _compare(w, cuda_device)
    ref_slots, kb, vb, ref, ref_err, valid = oracle_full(w, host)
    assert errbits == 0 and ref_err == set()
    assert np.array_equal(slots.cpu().numpy(), ref_slots)
    assert np.array_equal(bits(b["k_cache"]), kb) and np.array_equal(bits(b["v_cache"]), vb)
    assert_close(f64(out)[valid], ref[valid], w.dtype, w.name)


@pytest.mark.parametrize("n", [64, 4095, 4096, 4097, 6000])
def test_batch_sizes_across_the_planner_paths(cuda_device, n):
    """Up to 4096 requests the planner takes its one-pass decode path, above
    it the general one; the write spans many CTAs either way."""
    rng = np.random.default_rng(n)
    lens = rng.integers(1, 200, n).astype(np.int32)
    w = W.custom(f"dstep_n{n}", lens, np.ones(n, np.int32), 8, 2, 64, 16, "bf16", seed=n)
    _compare(w, cuda_device)


def test_llama8b_shapes_bf16_output(cuda_device):
    w = W.llama8b_decode(seed=5, num_seqs=16, min_len=100, max_len=1500)
    _compare(w, cuda_device, out_dtype=torch.bfloat16)


def test_fp8_pools(cuda_device):
    lens = [40, 300, 77, 1, 2000]
    w = W.with_fp8_cache(W.custom("dstep_fp8", lens, [1] * len(lens), 32, 8, 128, 16, "bf16",
                                  seed=91))
    _compare(w, cuda_device)


def test_shared_prefix_cascade(cuda_device):
    """40 requests whose tables start with the same 38 blocks: the planner
    sends the prefix to tensor-core tiles; the write goes to each suffix."""
    rng = np.random.default_rng(8)
    n, pblocks, bs = 40, 38, 16
    suffixes = rng.integers(1, 300, size=n)
    sblocks = (suffixes + bs - 1) // bs
    nb = pblocks + int(sblocks.sum()) + 3
    order = rng.permutation(nb).astype(np.int32)
    tables = np.full((n, pblocks + int(sblocks.max())), -1, np.int32)
    tables[:, :pblocks] = order[:pblocks]
    c = pblocks
    for i, m in enumerate(sblocks):
        tables[i, pblocks:pblocks + m] = order[c:c + m]
        c += m
    lens = (pblocks * bs + suffixes).astype(np.int32)
    w = W.custom("dstep_prefix", lens, np.ones(n, np.int32), 32, 8, 128, bs, "bf16", seed=8)
    w.block_tables, w.num_blocks = tables, nb
    host, b, out, slots, errbits = _compare(w, cuda_device)
    ref_slots, kb, vb, ref, ref_err, valid = oracle_full(w, host)
    assert errbits == 0
    assert np.array_equal(slots.cpu().numpy(), ref_slots)
    assert_close(f64(out)[valid], ref[valid], w.dtype, w.name)


def test_error_bits_match_the_two_calls(cuda_device):
    """A block id outside the pool, a seq_len longer than the table and a zero
    seq_len: the same bits, slots (-1), pools and written rows as the two
    calls."""
    dev = cuda_device
    w = W.custom("dstep_err", [20, 20, 20, 20, 20], [1] * 5, 8, 2, 64, 16, "f32", seed=15,
                 extra_blocks=1)
    idx = W.index_tensors(w, dev)
    idx["block_tables"][1, 1] = w.num_blocks + 5    # request 1's token (position 19)
    idx["seq_lens"][2] = 20 + 16 * 5                # request 2: longer than its table
    idx["seq_lens"][3] = 0                          # request 3: no token to place
    _, _, _, slots, errbits = _compare(w, dev, idx=idx)
    assert errbits == (P.ERRBIT_BLOCK_OOB | P.ERRBIT_SEQ_TOO_LONG | P.ERRBIT_QUERY_TOO_LONG)
    assert slots.cpu().tolist()[1:4] == [-1, -1, -1]


def test_determinism(cuda_device):
    dev = cuda_device
    lens = [900, 3000, 17, 250]
    w = W.custom("dstep_det", lens, [1] * len(lens), 32, 8, 128, 16, "bf16", seed=21)
    host = W.make_tensors(w, "cpu", where="host")
    idx = W.index_tensors(w, dev)
    outs = []
    for _ in range(3):
        t = _copies(host, dev)
        out, _ = _one_call(w, t, idx, P.new_error_word(dev), torch.float32)
        outs.append(bits(out))
    assert all(np.array_equal(outs[0], o) for o in outs[1:])


def test_shape_checks(cuda_device):
    dev = cuda_device
    w = W.custom("dstep_shape", [20, 30], [1, 1], 8, 2, 64, 16, "f32", seed=2)
    t = _copies(W.make_tensors(w, "cpu", where="host"), dev)
    idx = W.index_tensors(w, dev)
    k3 = torch.cat([t["k_new"], t["k_new"][:1]])
    with pytest.raises(ValueError):
        P.decode_step(t["q"], k3, t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
                      idx["seq_lens"], w.scale)
    with pytest.raises(ValueError):
        P.decode_step(t["q"], t["k_new"], t["v_new"].to(torch.bfloat16), t["k_cache"],
                      t["v_cache"], idx["block_tables"], idx["seq_lens"], w.scale)

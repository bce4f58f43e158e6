"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on the
same seeded inputs.  Cache writes and slots are compared bit for bit;
attention within max-abs 1e-5 (fp32) or max-abs 1e-2 / mean-abs 1e-3 (bf16
inputs, fp32 accumulation)."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import workloads as W

from _util import assert_close, bits, device_blocks, f64, oracle_full, oracle_request

pytestmark = pytest.mark.gpu


def _run(w, dev, out_dtype=torch.float32, host=None, err=None):
    host = host or W.make_tensors(w, "cpu", where="host")
    t = {k: v.to(dev) for k, v in host.items()}
    idx = W.index_tensors(w, dev)
    err = err if err is not None else P.new_error_word(dev)
    slots = torch.empty(w.num_tokens, dtype=torch.int64, device=dev)
    out = P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
                 idx["query_start_loc"], idx["seq_lens"], w.scale, decode_only=w.is_decode,
                 out_dtype=out_dtype, slots=slots, err=err)
    torch.cuda.synchronize()
    return host, t, slots, out, P.read_error(err)


def _check_all(w, dev, out_dtype=torch.float32):
    host, t, slots, out, errbits = _run(w, dev, out_dtype)
    ref_slots, kb, vb, ref, ref_err, valid = oracle_full(w, host)
    assert errbits == 0 and ref_err == set()
    assert np.array_equal(slots.cpu().numpy(), ref_slots)
    assert np.array_equal(bits(t["k_cache"]), kb)
    assert np.array_equal(bits(t["v_cache"]), vb)
    got = f64(out)
    if out_dtype == torch.bfloat16:
        # the oracle rounded to bf16 (RNE), plus half an ulp of bf16 at the value
        ref_r = torch.from_numpy(ref).to(torch.bfloat16).to(torch.float64).numpy()
        half_ulp = np.abs(ref_r) * 2.0 ** -8
        err = np.abs(got - ref_r)
        assert np.all(err <= 1e-2 + half_ulp)
        return
    return assert_close(got[valid], ref[valid], w.dtype, w.name)


def test_tiny_decode_fp32(cuda_device):
    _check_all(W.tiny_decode(0), cuda_device)


@pytest.mark.parametrize("seed", [1, 2])
def test_tiny_decode_fp32_other_seeds(cuda_device, seed):
    _check_all(W.tiny_decode(seed), cuda_device)


def _ragged_lens(bs, rng, n=9, longest=700):
    base = [1, bs - 1, bs, bs + 1, 2 * bs + 3, longest]
    extra = rng.integers(1, longest, size=max(0, n - len(base))).tolist()
    return [max(1, x) for x in base + extra]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (16, 2), (32, 8)])
def test_decode_random_shapes(cuda_device, dtype, bs, D, hq, hkv):
    rng = np.random.default_rng(bs * 1000 + D + hq)
    lens = _ragged_lens(bs, rng)
    w = W.custom(f"rand_decode_{dtype}", lens, np.ones(len(lens), np.int32), hq, hkv, D, bs,
                 dtype, seed=bs + D + hq, extra_blocks=3)
    _check_all(w, cuda_device)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("D", [64, 128])
def test_mixed_random_shapes(cuda_device, dtype, bs, D):
    rng = np.random.default_rng(7 * bs + D)
    # prefill chunks with and without a cached prefix, decodes, a chunk equal to its request
    lens = [70, 33, 1, bs, 130, 17, 200, 9]
    qlens = [20, 33, 1, 1, 64, 1, 3, 9]
    order = rng.permutation(len(lens))
    w = W.custom(f"rand_mixed_{dtype}", np.array(lens)[order], np.array(qlens)[order], 8, 2, D,
                 bs, dtype, seed=bs + D, extra_blocks=2)
    _check_all(w, cuda_device)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 4), (32, 2)])
@pytest.mark.parametrize("D", [64, 128])
def test_mixed_gqa_packings(cuda_device, hq, hkv, D):
    # prefill tiles pack 128/G tokens x G query heads; cover G = 1, 2, 8, 16,
    # chunks shorter and longer than a tile, a cached prefix not a multiple of 128
    lens = [300, 129, 1, 77, 520, 64]
    qlens = [150, 129, 1, 1, 8, 17]
    w = W.custom("mixed_gqa", lens, qlens, hq, hkv, D, 16, "bf16", seed=hq + hkv + D)
    _check_all(w, cuda_device)


def _shared_prefix_workload(name, n_seqs, prefix_blocks, suffixes, hq, hkv, d, bs, seed):
    """Decode batch whose block tables all start with the same physical blocks."""
    rng = np.random.default_rng(seed)
    sblocks = [(s + bs - 1) // bs for s in suffixes]
    nb = prefix_blocks + sum(sblocks) + 3
    order = rng.permutation(nb).astype(np.int32)
    width = prefix_blocks + max(sblocks)
    tables = np.full((n_seqs, width), -1, np.int32)
    tables[:, :prefix_blocks] = order[:prefix_blocks]
    c = prefix_blocks
    for b, n in enumerate(sblocks):
        tables[b, prefix_blocks:prefix_blocks + n] = order[c:c + n]
        c += n
    lens = (prefix_blocks * bs + np.asarray(suffixes)).astype(np.int32)
    w = W.custom(name, lens, np.ones(n_seqs, np.int32), hq, hkv, d, bs, "bf16", seed=seed)
    w.block_tables, w.num_blocks = tables, nb
    return w


@pytest.mark.parametrize("hq,hkv,d,bs", [(32, 8, 128, 16), (64, 8, 128, 32), (16, 8, 64, 16),
                                         (32, 2, 128, 8)])
def test_shared_prefix_cascade(cuda_device, hq, hkv, d, bs):
    # 40 requests share a prefix that is not a multiple of 128 keys; the prefix
    # is attended once by tensor-core tiles and merged with each suffix
    rng = np.random.default_rng(hq + bs)
    suffixes = rng.integers(1, 300, size=40).tolist()
    w = _shared_prefix_workload("prefix_cascade", 40, 600 // bs, suffixes, hq, hkv, d, bs, 17)
    _check_all(w, cuda_device)


def test_bf16_output_variant(cuda_device):
    w = W.custom("bf16_out", [5, 77, 300, 1], [1, 1, 1, 1], 32, 8, 128, 16, "bf16", seed=4)
    _check_all(w, cuda_device, out_dtype=torch.bfloat16)
    w = W.custom("bf16_out_mixed", [40, 77], [40, 1], 8, 2, 64, 16, "bf16", seed=5)
    _check_all(w, cuda_device, out_dtype=torch.bfloat16)


# ---------------------------------------------------------------- special cases

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_context_length_one_returns_v(cuda_device, dtype):
    w = W.custom("len1", [1, 1, 1], [1, 1, 1], 8, 2, 128, 16, dtype, seed=9)
    host, t, slots, out, errbits = _run(w, cuda_device)
    assert errbits == 0
    v = f64(host["v_new"])
    for b in range(3):
        for h in range(8):
            assert np.array_equal(f64(out)[b, h], v[b, h // 4])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_identical_keys_give_mean_of_v(cuda_device, dtype):
    L = 300
    w = W.custom("same_keys", [L], [1], 8, 2, 64, 16, dtype, seed=10)
    host = W.make_tensors(w, "cpu", where="host")
    host["k_cache"][:] = host["k_cache"][0, 0]
    host["k_new"][:] = host["k_cache"][0, 0]
    host2, t, slots, out, errbits = _run(w, cuda_device, host=host)
    _, _, _, ref, _, _ = oracle_full(w, host)
    # closed form: uniform weights -> the mean of the L value rows
    tables = w.block_tables[0]
    vv = oracle.cache_write(f64(host["v_cache"]), f64(host["v_cache"]), f64(host["v_new"]),
                            f64(host["v_new"]), oracle.slot_mapping(w.block_tables, [0, 1], [L], 16))[0]
    V = oracle.gather(vv, tables, L)
    for h in range(8):
        assert np.max(np.abs(ref[0, h] - V[:, h // 4].mean(0))) < 1e-12
    assert_close(f64(out)[0], ref[0], dtype, "identical keys")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_physical_block_permutation_is_bit_invariant(cuda_device, dtype):
    lens = [33, 500, 17, 1000]
    w1 = W.custom("perm_a", lens, [1] * 4, 32, 8, 128, 16, dtype, seed=11)
    host = W.make_tensors(w1, "cpu", where="host")
    _, _, _, out1, e1 = _run(w1, cuda_device, host=host)
    # same logical content under a different physical placement
    perm = np.random.default_rng(12).permutation(w1.num_blocks)
    w2 = W.custom("perm_b", lens, [1] * 4, 32, 8, 128, 16, dtype, seed=11)
    w2.block_tables = np.where(w1.block_tables >= 0, perm[np.maximum(w1.block_tables, 0)],
                               -1).astype(np.int32)
    host2 = dict(host)
    for name in ("k_cache", "v_cache"):
        moved = torch.empty_like(host[name])
        moved[torch.from_numpy(perm)] = host[name]
        host2[name] = moved
    _, _, _, out2, e2 = _run(w2, cuda_device, host=host2)
    assert e1 == e2 == 0
    assert torch.equal(out1, out2)


def test_zero_length_decode_row_is_zero(cuda_device):
    w = W.custom("zero_len", [5, 1, 40], [1, 1, 1], 8, 2, 64, 16, "bf16", seed=13)
    host = W.make_tensors(w, "cpu", where="host")
    t = {k: v.to(cuda_device) for k, v in host.items()}
    lens = torch.tensor([5, 0, 40], dtype=torch.int32, device=cuda_device)
    tables = torch.from_numpy(w.block_tables).to(cuda_device)
    out = torch.full((3, 8, 64), float("nan"), device=cuda_device)
    P.decode(t["q"], t["k_cache"], t["v_cache"], tables, lens, w.scale, out=out)
    torch.cuda.synchronize()
    assert torch.all(out[1] == 0)
    ref, err, valid = oracle.paged_decode(f64(host["q"]), f64(host["k_cache"]),
                                          f64(host["v_cache"]), w.block_tables,
                                          np.array([5, 0, 40]), w.scale)
    assert_close(f64(out), ref, "bf16", "zero-length row")


def test_determinism(cuda_device):
    w = W.custom("det", [4000, 33, 1234], [1, 1, 1], 32, 8, 128, 16, "bf16", seed=14)
    _, _, _, a, _ = _run(w, cuda_device)
    _, _, _, b, _ = _run(w, cuda_device)
    assert torch.equal(a, b)


@pytest.mark.parametrize("lens", [[1200, 40], [4000, 9], [1200, 4000, 17]])
def test_merge_paths_by_partition_count(cuda_device, lens):
    """Rows split into 33 to 64 partitions reach the per-warp merge's second
    chunk of partitions; rows with more reach the per-CTA merge.  (In these
    small batches the planner cuts a 1200-key row into 38 pieces and a
    4000-key row into 125: two-stage pieces over most of the row, then
    smaller ones.)"""
    w = W.custom("merge_paths", lens, [1] * len(lens), 32, 8, 128, 16, "bf16", seed=31)
    _check_all(w, cuda_device)


# ---------------------------------------------------------------- device errors

def test_error_bits_bad_inputs(cuda_device):
    dev = cuda_device
    w = W.custom("errs", [20, 20, 20], [1, 1, 1], 8, 2, 64, 16, "f32", seed=15, extra_blocks=1)
    host = W.make_tensors(w, "cpu", where="host")
    t = {k: v.to(dev) for k, v in host.items()}
    tables = torch.from_numpy(w.block_tables).to(dev)
    err = P.new_error_word(dev)
    sentinel = -7.0

    # block id outside the pool: that row is left unwritten, others are fine
    bad = tables.clone()
    bad[1, 0] = w.num_blocks + 5
    out = torch.full((3, 8, 64), sentinel, device=dev)
    P.decode(t["q"], t["k_cache"], t["v_cache"], bad, torch.from_numpy(w.seq_lens).to(dev),
             w.scale, out=out, err=err)
    assert P.read_error(err) == P.ERRBIT_BLOCK_OOB
    assert torch.all(out[1] == sentinel) and not torch.any(out[0] == sentinel)

    # seq_len longer than the table
    lens = torch.tensor([20, 20 + 16 * 5, 20], dtype=torch.int32, device=dev)
    out.fill_(sentinel)
    P.decode(t["q"], t["k_cache"], t["v_cache"], tables, lens, w.scale, out=out, err=err)
    assert P.read_error(err) == P.ERRBIT_SEQ_TOO_LONG
    assert torch.all(out[1] == sentinel) and not torch.any(out[2] == sentinel)

    # query longer than its sequence (mixed step)
    qsl = torch.tensor([0, 1, 3, 3], dtype=torch.int32, device=dev)
    lens2 = torch.tensor([20, 1, 20], dtype=torch.int32, device=dev)
    out.fill_(sentinel)
    P.mixed_step(t["q"], t["k_cache"], t["v_cache"], tables, qsl, lens2, w.scale, out=out, err=err)
    assert P.read_error(err) == P.ERRBIT_QUERY_TOO_LONG
    assert torch.all(out[1:3] == sentinel) and not torch.any(out[0] == sentinel)

    # slot outside the pool (skipped) and negative slot (padding, silent)
    before_k = t["k_cache"].clone()
    slots = torch.tensor([-1, w.num_blocks * 16, 5], dtype=torch.int64, device=dev)
    P.cache_write(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], slots, err=err)
    assert P.read_error(err) == P.ERRBIT_SLOT_OOB
    changed = (t["k_cache"] != before_k).reshape(-1, 2 * 64).any(1).nonzero().flatten().tolist()
    assert changed == [5]


# ---------------------------------------------------------------- full-size workloads

def _full_size(w, dev, reqs, out_dtype=torch.float32):
    """Run a full-size workload through the step; check slots and cache writes
    by properties that hold at any size, and EVERY output row of the requests
    in `reqs` against the oracle, element by element."""
    t = W.make_tensors(w, dev, where="device")
    idx = W.index_tensors(w, dev)
    blocks = device_blocks(w, (t["k_cache"], t["v_cache"]), reqs)
    # untouched-slot sample, taken before the step
    gen = np.random.default_rng(99)
    probe = torch.from_numpy(gen.integers(0, w.num_blocks * w.block_size, 4096)).to(dev)
    kc_flat = t["k_cache"].view(-1, w.num_kv_heads, w.head_dim)
    before = kc_flat.index_select(0, probe).clone()
    err = P.new_error_word(dev)
    slots = torch.empty(w.num_tokens, dtype=torch.int64, device=dev)
    out = P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
                 idx["query_start_loc"], idx["seq_lens"], w.scale, decode_only=w.is_decode,
                 out_dtype=out_dtype, slots=slots, err=err)
    torch.cuda.synchronize()
    assert P.read_error(err) == 0
    # slots: bit-exact against the oracle's slot function
    ref_slots = oracle.slot_mapping(w.block_tables, w.query_start_loc, w.seq_lens, w.block_size)
    assert np.array_equal(slots.cpu().numpy(), ref_slots)
    # every written row holds the new token's row, bit for bit
    assert torch.equal(kc_flat.index_select(0, slots), t["k_new"])
    vc_flat = t["v_cache"].view(-1, w.num_kv_heads, w.head_dim)
    assert torch.equal(vc_flat.index_select(0, slots), t["v_new"])
    # rows that were not written are unchanged
    written = set(ref_slots.tolist())
    keep = torch.tensor([i for i, s in enumerate(probe.tolist()) if s not in written], device=dev)
    assert torch.equal(kc_flat.index_select(0, probe)[keep], before[keep])
    # attention: every row of the chosen requests
    k_new, v_new, q = t["k_new"].cpu(), t["v_new"].cpu(), t["q"].cpu()
    qsl = w.query_start_loc
    got, ref = [], []
    for b in reqs:
        ref.append(oracle_request(w, blocks.pop(int(b)), k_new, v_new, q, int(b)))
        got.append(f64(out[int(qsl[b]):int(qsl[b + 1])]))
    return assert_close(np.concatenate(got), np.concatenate(ref), w.dtype, w.name), out


def test_full_llama8b_decode(cuda_device):
    w = W.llama8b_decode(0)
    _full_size(w, cuda_device, range(w.num_seqs))          # all 64 requests


def test_full_long_context_split_kv(cuda_device):
    _full_size(W.long_context_decode(0), cuda_device, [0, 1, 2, 3])


def test_full_shared_prefix_decode(cuda_device):
    w = W.shared_prefix_decode(0)
    _full_size(w, cuda_device, range(w.num_seqs))          # all 128 requests


def _mixed_requests(w, n_decode=256, seed=7):
    """Both prefill chunks (every one of their 4096 rows) and n_decode decode
    requests drawn by a seeded generator."""
    big = [b for b in range(w.num_seqs) if w.query_lens[b] > 1]
    dec = [b for b in range(w.num_seqs) if w.query_lens[b] == 1]
    pick = np.random.default_rng(seed).choice(dec, size=n_decode, replace=False)
    return sorted(big + [int(b) for b in pick])


@pytest.mark.late(1)
def test_full_mixed_step(cuda_device):
    w = W.mixed_step(0)
    reqs = _mixed_requests(w)
    assert sum(int(w.query_lens[b]) for b in reqs) == 4096 + 256
    _full_size(w, cuda_device, reqs)


@pytest.mark.late(1)
def test_full_mixed_step_shuffled(cuda_device):
    w = W.mixed_step(1, shuffle=True)
    _full_size(w, cuda_device, _mixed_requests(w, seed=8))

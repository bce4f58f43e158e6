"""Copy-on-write block copies and the slot build from (request, position):
the CUDA path against the oracle (oracle/blocks.py), bit-exact."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_434_b200 as P
from _util import bits

pytestmark = pytest.mark.gpu


def _pools(nb, bs, hkv, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    return (torch.randn(nb, bs, hkv, d, generator=g).to(td),
            torch.randn(nb, bs, hkv, d, generator=g).to(td))


def _pairs(nb, n, rng, bad=0):
    ids = rng.permutation(nb)
    src, dst = ids[:n], ids[n:2 * n]               # no block is both a source and a destination
    m = np.stack([src, dst], axis=1).astype(np.int64)
    for i in range(bad):
        m[rng.integers(n), rng.integers(2)] = nb + int(rng.integers(5))
    return m


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("nb,bs,hkv,d", [(40, 16, 8, 128), (33, 8, 2, 64), (20, 32, 1, 128),
                                         (64, 16, 4, 64)])
def test_copy_blocks_parity(cuda_device, dtype, nb, bs, hkv, d):
    rng = np.random.default_rng([nb, bs, hkv, d])
    kp, vp = _pools(nb, bs, hkv, d, dtype, nb + d)
    m = _pairs(nb, nb // 3, rng, bad=1)
    kd, vd = kp.to(cuda_device), vp.to(cuda_device)
    err = P.new_error_word(cuda_device)
    P.copy_blocks(kd, vd, torch.from_numpy(m).to(cuda_device), err=err)
    torch.cuda.synchronize()
    kr, vr, errs = oracle.copy_blocks(bits(kp), bits(vp), m)
    assert np.array_equal(bits(kd), kr) and np.array_equal(bits(vd), vr)
    assert P.read_error(err) == P.ERRBIT_BLOCK_OOB and errs == {oracle.ERR_BLOCK_OOB}


def test_copy_blocks_full_size(cuda_device):
    """2048 copy-on-write pairs in Llama-3-8B layer pools (block 16 x 8 heads x
    128, bf16: 32 KiB per block and pool)."""
    nb = 8192
    kp, vp = _pools(nb, 16, 8, 128, "bf16", 11)
    kd, vd = kp.to(cuda_device), vp.to(cuda_device)
    m = _pairs(nb, 2048, np.random.default_rng(12))
    P.copy_blocks(kd, vd, torch.from_numpy(m).to(cuda_device))
    torch.cuda.synchronize()
    src, dst = torch.from_numpy(m[:, 0]), torch.from_numpy(m[:, 1])
    assert torch.equal(kd.cpu()[dst].view(torch.int16), kp[src].view(torch.int16))
    assert torch.equal(vd.cpu()[dst].view(torch.int16), vp[src].view(torch.int16))
    keep = torch.ones(nb, dtype=torch.bool)
    keep[dst] = False
    assert torch.equal(kd.cpu()[keep].view(torch.int16), kp[keep].view(torch.int16))


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_slot_mapping_positions_parity(cuda_device, bs):
    rng = np.random.default_rng([bs, 5])
    nb, B, W, T = 200, 7, 24, 500
    tables = rng.permutation(nb)[:B * W].reshape(B, W).astype(np.int32)
    tables[2, 10:] = -1                                  # unused tail of a table
    tables[4, 3] = nb + 7                                # a bad entry
    req = rng.integers(-1, B + 1, T).astype(np.int32)    # -1 padding, B out of range
    pos = rng.integers(-2, W * bs + 3, T).astype(np.int64)
    err = P.new_error_word(cuda_device)
    out = P.slot_mapping_positions(torch.from_numpy(tables).to(cuda_device),
                                   torch.from_numpy(req).to(cuda_device),
                                   torch.from_numpy(pos).to(cuda_device), bs, nb, err=err)
    torch.cuda.synchronize()
    ref, errs = oracle.slot_mapping_positions(tables, req, pos, bs, nb)
    assert np.array_equal(out.cpu().numpy(), ref)
    want = (P.ERRBIT_POS_OOB if oracle.ERR_POS_OOB_TABLE in errs else 0) | \
           (P.ERRBIT_BLOCK_OOB if oracle.ERR_BLOCK_OOB in errs else 0)
    assert P.read_error(err) == want and want == P.ERRBIT_POS_OOB | P.ERRBIT_BLOCK_OOB


def test_slot_mapping_positions_matches_step_slots(cuda_device):
    """For the tokens of a flattened step (the last q_b positions of each
    request) both slot builders agree bit for bit."""
    from paged_kv_cache_434_b200 import workloads as W
    w = W.mixed_step(0)
    idx = W.index_tensors(w, cuda_device)
    a = P.slot_mapping(idx["block_tables"], idx["query_start_loc"], idx["seq_lens"], w.block_size,
                       w.num_blocks, w.num_tokens)
    req = np.repeat(np.arange(w.num_seqs), w.query_lens).astype(np.int32)
    pos = np.concatenate([np.arange(w.seq_lens[b] - w.query_lens[b], w.seq_lens[b])
                          for b in range(w.num_seqs)]).astype(np.int64)
    b = P.slot_mapping_positions(idx["block_tables"], torch.from_numpy(req).to(cuda_device),
                                 torch.from_numpy(pos).to(cuda_device), w.block_size, w.num_blocks)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_copy_on_write_fork_through_attention(cuda_device):
    """Request A forks into B; B appends a token into the shared, partly filled
    last block after copying it.  A's decode output is bit-identical before
    and after, B's matches the oracle."""
    from _util import f64
    dev = cuda_device
    rng = np.random.default_rng(21)
    bs, nb, hq, hkv, d = 16, 12, 8, 2, 64
    kp, vp = _pools(nb, bs, hkv, d, "f32", 22)
    kd, vd = kp.to(dev), vp.to(dev)
    L = 37                                               # 3 blocks, the last holds 5 tokens
    table_a = np.array([7, 2, 9], dtype=np.int32)
    q = torch.from_numpy(rng.standard_normal((1, hq, d), dtype=np.float32)).to(dev)
    lens = torch.tensor([L], dtype=torch.int32, device=dev)
    ta = torch.from_numpy(table_a[None]).to(dev)
    before = P.decode(q, kd, vd, ta, lens, 0.125).cpu()
    # fork: B shares A's blocks; its write into block 9 needs a copy first
    table_b = table_a.copy()
    table_b[2] = 4
    P.copy_blocks(kd, vd, torch.tensor([[9, 4]], dtype=torch.int64, device=dev))
    tb = torch.from_numpy(table_b[None]).to(dev)
    slots = P.slot_mapping_positions(tb, torch.zeros(1, dtype=torch.int32, device=dev),
                                     torch.tensor([L], dtype=torch.int64, device=dev), bs, nb)
    k_new = torch.from_numpy(rng.standard_normal((1, hkv, d), dtype=np.float32)).to(dev)
    v_new = torch.from_numpy(rng.standard_normal((1, hkv, d), dtype=np.float32)).to(dev)
    P.cache_write(k_new, v_new, kd, vd, slots)
    after = P.decode(q, kd, vd, ta, lens, 0.125).cpu()
    out_b = P.decode(q, kd, vd, tb, lens + 1, 0.125).cpu()
    torch.cuda.synchronize()
    assert np.array_equal(bits(after), bits(before))
    kr, vr, _ = oracle.copy_blocks(f64(kp), f64(vp), [[9, 4]])
    kr, vr, _ = oracle.cache_write(kr, vr, f64(k_new.cpu()), f64(v_new.cpu()),
                                   np.array([oracle.slot_of(table_b, L, bs)]))
    ref, _, _ = oracle.paged_decode(f64(q.cpu()), kr, vr, table_b[None], np.array([L + 1]), 0.125)
    assert np.abs(f64(out_b) - ref).max() <= 1e-5

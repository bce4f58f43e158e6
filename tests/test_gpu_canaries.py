"""Canary words around every buffer the library writes.

Each output of a call (pools, slots, attention output, workspace, rotated
queries, the cos/sin table) is carved out of a larger device buffer whose
GUARD bytes on either side hold a fixed byte pattern.  After the call, the
pattern must be intact: no kernel writes before or after the buffer it was
given, even when the workspace is exactly the size the library asked for.
The results inside are checked against the oracle as in the parity suites.

The `late` mark runs this file after the other GPU tests except the no-alloc ones.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import workloads as W
from _util import assert_close, bits, f64, fp8_codes, oracle_full, oracle_full_fp8

pytestmark = [pytest.mark.gpu, pytest.mark.late(3)]

GUARD = 4096   # bytes on each side; a multiple of 256 keeps the inner buffer 256-byte aligned
FILL = 0xA5


class Guarded:
    """`nbytes` of device memory between two GUARD-byte canary regions."""

    def __init__(self, nbytes, dev):
        self.nbytes = int(nbytes)
        self.raw = torch.full((2 * GUARD + self.nbytes,), FILL, dtype=torch.uint8, device=dev)

    def tensor(self, dtype, shape):
        return self.raw[GUARD:GUARD + self.nbytes].view(dtype).view(shape)

    def intact(self) -> bool:
        return bool((self.raw[:GUARD] == FILL).all()) and \
            bool((self.raw[GUARD + self.nbytes:] == FILL).all())


def guarded_copy(t, dev):
    g = Guarded(t.numel() * t.element_size(), dev)
    x = g.tensor(t.dtype, tuple(t.shape))
    x.copy_(t.to(dev))
    return g, x


def guarded_empty(dtype, shape, dev):
    elt = torch.empty((), dtype=dtype).element_size()
    g = Guarded(int(np.prod(shape)) * elt, dev)
    return g, g.tensor(dtype, tuple(shape))


def assert_intact(what, **guards):
    for name, g in guards.items():
        assert g.intact(), f"{what}: a write landed outside {name}"


def test_guard_detects_a_stray_byte():
    g = Guarded(64, "cpu")
    assert g.intact()
    g.raw[GUARD + 64] = 0
    assert not g.intact()


# ---------------------------------------------------------------- attention steps

def _attention_step(w, dev, out_dtype=torch.float32):
    host = W.make_tensors(w, "cpu", where="host")
    idx = W.index_tensors(w, dev)
    q, k_new, v_new = (host[n].to(dev) for n in ("q", "k_new", "v_new"))
    gk, kc = guarded_copy(host["k_cache"], dev)
    gv, vc = guarded_copy(host["v_cache"], dev)
    T, Hq, D = w.num_tokens, w.num_heads, w.head_dim
    B, width = w.block_tables.shape
    gs, slots = guarded_empty(torch.int64, (T,), dev)
    go, out = guarded_empty(out_dtype, (T, Hq, D), dev)
    nbytes = (P.decode_workspace_size(B, Hq, width, kc) if w.is_decode else
              P.mixed_step_workspace_size(B, T, Hq, width, kc))
    assert nbytes > 0
    gw, ws = guarded_empty(torch.uint8, (nbytes,), dev)
    err = P.new_error_word(dev)
    P.step(q, k_new, v_new, kc, vc, idx["block_tables"], idx["query_start_loc"], idx["seq_lens"],
           w.scale, decode_only=w.is_decode, out=out, out_dtype=out_dtype, slots=slots,
           workspace=ws, err=err, kv_scales=w.kv_scales)
    torch.cuda.synchronize()
    assert P.read_error(err) == 0
    assert_intact(w.name, k_cache=gk, v_cache=gv, slots=gs, out=go, workspace=gw)
    return host, kc, vc, slots, out


def _check_against_oracle(w, host, kc, vc, slots, out):
    if w.kv_dtype == "fp8":
        ref_slots, kb, vb, ref, ref_err, valid = oracle_full_fp8(w, host)
        assert np.array_equal(fp8_codes(kc), kb) and np.array_equal(fp8_codes(vc), vb)
    else:
        ref_slots, kb, vb, ref, ref_err, valid = oracle_full(w, host)
        assert np.array_equal(bits(kc), kb) and np.array_equal(bits(vc), vb)
    assert ref_err == set()
    assert np.array_equal(slots.cpu().numpy(), ref_slots)
    assert_close(f64(out)[valid], ref[valid], "bf16" if w.dtype == "bf16" else "f32", w.name)


ATTENTION_CASES = {
    # fp32 pools: the generic kernel
    "fp32_decode": lambda: W.tiny_decode(0),
    # bf16 Llama-3-8B heads: TMA-staged mma.sync partitions, split-KV, merge
    "bf16_decode_split": lambda: W.custom("canary_dec", [1, 15, 16, 17, 700, 3000, 5000],
                                          [1] * 7, 32, 8, 128, 16, "bf16", seed=21,
                                          extra_blocks=3),
    # head_dim 64, block size 8: per-head TMA boxes
    "bf16_decode_d64_bs8": lambda: W.custom("canary_dec_d64", [3, 8, 9, 400, 1200], [1] * 5,
                                            8, 2, 64, 8, "bf16", seed=22, extra_blocks=2),
    # chunked prefill + decodes: tcgen05 tiles beside the decode partitions
    "bf16_mixed": lambda: W.custom("canary_mixed", [300, 17, 1024, 5, 700], [1, 9, 200, 1, 64],
                                   32, 8, 128, 16, "bf16", seed=23),
    "bf16_mixed_d64": lambda: W.custom("canary_mixed_d64", [130, 40, 600], [130, 1, 77],
                                       8, 2, 64, 16, "bf16", seed=24),
    # 32 requests over a shared 512-token prefix: tensor-core prefix tiles
    # writing split-KV partials, suffix partitions, merge
    "bf16_shared_prefix": lambda: W.shared_prefix_decode(3, num_seqs=32, prefix_tokens=512),
    # e4m3 pools
    "fp8_decode": lambda: W.with_fp8_cache(W.custom("canary_fp8", [1, 16, 17, 900, 2500],
                                                    [1] * 5, 32, 8, 128, 16, "bf16", seed=25)),
    "fp8_mixed": lambda: W.with_fp8_cache(W.custom("canary_fp8_mixed", [300, 17, 700],
                                                   [1, 9, 64], 32, 8, 128, 16, "bf16", seed=26)),
}


@pytest.mark.parametrize("case", sorted(ATTENTION_CASES))
def test_attention_step_stays_in_its_buffers(cuda_device, case):
    w = ATTENTION_CASES[case]()
    host, kc, vc, slots, out = _attention_step(w, cuda_device)
    _check_against_oracle(w, host, kc, vc, slots, out)


def test_bf16_output_stays_in_its_buffer(cuda_device):
    w = ATTENTION_CASES["bf16_mixed"]()
    _, _, _, _, out = _attention_step(w, cuda_device, out_dtype=torch.bfloat16)
    assert torch.isfinite(out.float()).all()


def test_decode_no_alloc_stays_in_its_buffer(cuda_device):
    dev = cuda_device
    w = ATTENTION_CASES["bf16_decode_split"]()
    host = W.make_tensors(w, "cpu", where="host")
    idx = W.index_tensors(w, dev)
    t = {k: v.to(dev) for k, v in host.items()}
    go, out = guarded_empty(torch.float32, (w.num_seqs, w.num_heads, w.head_dim), dev)
    err = P.new_error_word(dev)
    P.decode_no_alloc(t["q"], t["k_cache"], t["v_cache"], idx["block_tables"], idx["seq_lens"],
                      w.scale, out, err=err)
    torch.cuda.synchronize()
    assert P.read_error(err) == 0
    assert_intact(w.name, out=go)
    # the pools were not written: every key, the last included, is history
    ref, _, valid = oracle.paged_mixed_step(f64(host["q"]), f64(host["k_cache"]),
                                            f64(host["v_cache"]), w.block_tables,
                                            w.query_start_loc, w.seq_lens, w.scale)
    assert_close(f64(out)[valid], ref[valid], "bf16", w.name)


# ---------------------------------------------------------------- next-row entry points

def test_rope_cache_write_stays_in_its_buffers(cuda_device):
    dev = cuda_device
    T, hq, hkv, d, nb, bs, max_pos, rot = 37, 32, 8, 128, 9, 16, 4096, 128
    rng = np.random.default_rng([31, 77])
    mk = lambda *s: torch.from_numpy(rng.standard_normal(s, dtype=np.float32)).to(torch.bfloat16)
    q, k, v = mk(T, hq, d), mk(T, hkv, d), mk(T, hkv, d)
    kp, vp = mk(nb, bs, hkv, d), mk(nb, bs, hkv, d)
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    pos = rng.integers(0, max_pos, T).astype(np.int64)
    gt, table = guarded_empty(torch.float32, (max_pos, rot), dev)
    P.rope_cos_sin_cache(max_pos, rot, 500000.0, out=table)
    gk, kc = guarded_copy(kp, dev)
    gv, vc = guarded_copy(vp, dev)
    gq, q_out = guarded_empty(torch.bfloat16, (T, hq, d), dev)
    err = P.new_error_word(dev)
    P.rope_cache_write(q.to(dev), k.to(dev), v.to(dev), kc, vc, torch.from_numpy(slots).to(dev),
                       torch.from_numpy(pos).to(dev), table, neox=True, q_out=q_out, err=err)
    torch.cuda.synchronize()
    assert P.read_error(err) == 0
    assert_intact("rope", cos_sin_cache=gt, k_cache=gk, v_cache=gv, q_out=gq)
    # V rows are stored unchanged: bit for bit at their slots, all else untouched
    exp_k, exp_v, _ = oracle.cache_write(bits(kp), bits(vp), bits(k), bits(v), slots)
    assert np.array_equal(bits(vc), exp_v)
    written = np.zeros(nb * bs, bool)
    written[slots] = True
    assert np.array_equal(bits(kc).reshape(nb * bs, -1)[~written],
                          exp_k.reshape(nb * bs, -1)[~written])


def test_copy_blocks_stays_in_its_buffers(cuda_device):
    dev = cuda_device
    nb, bs, hkv, d = 12, 16, 8, 128
    rng = np.random.default_rng(41)
    kp = torch.from_numpy(rng.standard_normal((nb, bs, hkv, d), dtype=np.float32)).to(torch.bfloat16)
    vp = torch.from_numpy(rng.standard_normal((nb, bs, hkv, d), dtype=np.float32)).to(torch.bfloat16)
    ids = rng.permutation(nb)
    pairs = np.stack([ids[:4], ids[4:8]], axis=1).astype(np.int64)
    gk, kc = guarded_copy(kp, dev)
    gv, vc = guarded_copy(vp, dev)
    err = P.new_error_word(dev)
    P.copy_blocks(kc, vc, torch.from_numpy(pairs).to(dev), err=err)
    torch.cuda.synchronize()
    assert P.read_error(err) == 0
    assert_intact("copy_blocks", k_cache=gk, v_cache=gv)
    exp_k, exp_v, errs = oracle.copy_blocks(bits(kp), bits(vp), pairs)
    assert not errs
    assert np.array_equal(bits(kc), exp_k) and np.array_equal(bits(vc), exp_v)


def test_slot_mapping_positions_stays_in_its_buffer(cuda_device):
    dev = cuda_device
    w = ATTENTION_CASES["bf16_decode_split"]()
    rng = np.random.default_rng(51)
    T = 300
    req = rng.integers(0, w.num_seqs, T).astype(np.int32)
    pos = np.array([rng.integers(0, w.seq_lens[b]) for b in req], dtype=np.int64)
    idx = W.index_tensors(w, dev)
    gs, out = guarded_empty(torch.int64, (T,), dev)
    err = P.new_error_word(dev)
    P.slot_mapping_positions(idx["block_tables"], torch.from_numpy(req).to(dev),
                             torch.from_numpy(pos).to(dev), w.block_size, w.num_blocks, out=out,
                             err=err)
    torch.cuda.synchronize()
    assert P.read_error(err) == 0
    assert_intact("slot_mapping_positions", slots=gs)
    ref, errs = oracle.slot_mapping_positions(w.block_tables, req, pos, w.block_size,
                                              w.num_blocks)
    assert not errs
    assert np.array_equal(out.cpu().numpy(), ref)

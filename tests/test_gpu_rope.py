"""Rotary embedding fused with the cache write: the CUDA path against the
fp64 oracle (oracle/rope.py) on the same seeded inputs."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_434_b200 as P
from _util import bits, f64

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5


def _tdtype(dtype):
    return torch.float32 if dtype == "f32" else torch.bfloat16


def _close(got, ref, dtype, what):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    if dtype == "f32":
        assert err.max() <= TOL_F32, (what, err.max())
    else:
        # one bf16 rounding of the float32 rotation: half an ulp of bf16 at a
        # value in [2^e, 2^(e+1)) is 2^(e-8) <= 2^-8 |value|
        bound = 2.0 ** -8 * np.abs(ref) * 1.001 + 1e-6
        assert np.all(err <= bound), (what, float((err - bound).max()))


@pytest.mark.parametrize("max_pos,rot,theta", [(4096, 128, 500000.0), (2048, 64, 10000.0),
                                               (131072, 128, 500000.0)])
def test_cos_sin_table(cuda_device, max_pos, rot, theta):
    got = P.rope_cos_sin_cache(max_pos, rot, theta, device=cuda_device).cpu().numpy()
    ref = oracle.cos_sin_table(max_pos, rot, theta).astype(np.float32)
    # the same float64 values rounded once: equal up to one float32 ulp
    assert np.abs(got.astype(np.float64) - ref).max() <= 2.0 ** -24 * 2


def _case(T, hq, hkv, d, nb, bs, dtype, seed, max_pos):
    rng = np.random.default_rng([seed, 77])
    td = _tdtype(dtype)
    mk = lambda *s: torch.from_numpy(rng.standard_normal(s, dtype=np.float32)).to(td)
    q, k, v = mk(T, hq, d), mk(T, hkv, d), mk(T, hkv, d)
    kp, vp = mk(nb, bs, hkv, d), mk(nb, bs, hkv, d)
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[rng.random(T) < 0.1] = -1                      # padding tokens
    pos = rng.integers(0, max_pos, T).astype(np.int64)
    return q, k, v, kp, vp, slots, pos


def _run(dev, q, k, v, kp, vp, slots, pos, table_gpu, neox, q_out=None):
    kp_d, vp_d = kp.to(dev), vp.to(dev)
    err = P.new_error_word(dev)
    out = P.rope_cache_write(q, k, v, kp_d, vp_d, torch.from_numpy(slots).to(dev),
                             torch.from_numpy(pos).to(dev), table_gpu, neox=neox, q_out=q_out,
                             err=err)
    torch.cuda.synchronize()
    return out.cpu(), kp_d.cpu(), vp_d.cpu(), P.read_error(err)


def _check(q, k, v, kp, vp, slots, pos, got, rot, neox, theta, max_pos, dtype):
    q_out, kp_g, vp_g, errbits = got
    table = oracle.cos_sin_table(max_pos, rot, theta)
    qr, kref, vref, errs, ok = oracle.rope_cache_write(f64(q), f64(k), f64(v), pos, slots, f64(kp),
                                                       f64(vp), table, rot, neox)
    _close(f64(q_out), qr, dtype, "q")
    nb, bs = kp.shape[:2]
    written = np.zeros((nb, bs), bool)
    for t, s in enumerate(slots):
        if 0 <= s < nb * bs and ok[t]:
            written[s // bs, s % bs] = True
    _close(f64(kp_g)[written], kref[written], dtype, "k rows")
    assert np.array_equal(bits(kp_g)[~written], bits(kp)[~written])     # untouched: bit-exact
    vb = bits(vp).copy()
    for t, s in enumerate(slots):
        if 0 <= s < nb * bs and ok[t]:
            vb[s // bs, s % bs] = bits(v)[t]
    assert np.array_equal(bits(vp_g), vb)                                # V: bit-exact copy
    return errbits, errs


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("neox", [True, False])
@pytest.mark.parametrize("d,rot", [(128, 128), (128, 64), (64, 64), (64, 32)])
def test_rope_cache_write_parity(cuda_device, dtype, neox, d, rot):
    dev = cuda_device
    theta, max_pos = 500000.0, 8192
    q, k, v, kp, vp, slots, pos = _case(37, 8, 2, d, 8, 16, dtype, d + rot + neox, max_pos)
    table = P.rope_cos_sin_cache(max_pos, rot, theta, device=dev)
    got = _run(dev, q.to(dev), k.to(dev), v.to(dev), kp, vp, slots, pos, table, neox)
    errbits, errs = _check(q, k, v, kp, vp, slots, pos, got, rot, neox, theta, max_pos, dtype)
    assert errbits == 0 and errs == set()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fused_qkv_slices_and_in_place(cuda_device, dtype):
    """q/k/v as column slices of one fused QKV output; queries rotated in place."""
    dev = cuda_device
    T, hq, hkv, d, rot, theta, max_pos = 53, 32, 8, 128, 128, 500000.0, 4096
    q, k, v, kp, vp, slots, pos = _case(T, hq, hkv, d, 16, 16, dtype, 5, max_pos)
    qkv = torch.cat([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], dim=1).to(dev)
    qs = qkv[:, :hq * d].view(T, hq, d)                   # strided views, no copy
    ks = qkv[:, hq * d:(hq + hkv) * d].view(T, hkv, d)
    vs = qkv[:, (hq + hkv) * d:].view(T, hkv, d)
    assert qs.stride(0) == (hq + 2 * hkv) * d
    table = P.rope_cos_sin_cache(max_pos, rot, theta, device=dev)
    got = _run(dev, qs, ks, vs, kp, vp, slots, pos, table, True)
    _check(q, k, v, kp, vp, slots, pos, got, rot, True, theta, max_pos, dtype)
    qc = q.to(dev).contiguous()
    got2 = _run(dev, qc, k.to(dev), v.to(dev), kp, vp, slots, pos, table, True, q_out=qc)
    assert np.array_equal(bits(got2[0]), bits(got[0]))     # in place == out of place
    assert np.array_equal(bits(qc.cpu()), bits(got[0]))


def test_bad_positions_and_slots(cuda_device):
    dev = cuda_device
    T, max_pos, rot, theta = 20, 64, 64, 10000.0
    q, k, v, kp, vp, slots, pos = _case(T, 4, 2, 64, 4, 16, "f32", 9, max_pos)
    slots = np.arange(T, dtype=np.int64)
    pos[3], pos[7] = max_pos, -5                          # outside the table
    slots[11] = 4 * 16                                    # past the pool
    table = P.rope_cos_sin_cache(max_pos, rot, theta, device=dev)
    got = _run(dev, q.to(dev), k.to(dev), v.to(dev), kp, vp, slots, pos, table, False)
    errbits, errs = _check(q, k, v, kp, vp, slots, pos, got, rot, False, theta, max_pos, "f32")
    assert errbits == P.ERRBIT_POS_OOB | P.ERRBIT_SLOT_OOB
    assert errs == {oracle.ERR_POS_OOB, "slot_out_of_range"}
    assert np.array_equal(bits(got[0][3]), bits(q[3]))    # copied unrotated


def test_full_size_mixed_step_tokens(cuda_device):
    """Llama-3-8B geometry, the 8192 new tokens of the mixed chunked-prefill
    step (positions of the two chunks and the decodes); sampled tokens
    against the oracle, every row's norm checked."""
    from paged_kv_cache_434_b200 import workloads as W
    dev = cuda_device
    w = W.mixed_step(0)
    T, hq, hkv, d = w.num_tokens, w.num_heads, w.num_kv_heads, w.head_dim
    qsl = w.query_start_loc
    pos = np.concatenate([np.arange(w.seq_lens[b] - w.query_lens[b], w.seq_lens[b])
                          for b in range(w.num_seqs)]).astype(np.int64)
    rng = np.random.default_rng([0, 78])
    nb, bs = 600, 16
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    mk = lambda *s: torch.from_numpy(rng.standard_normal(s, dtype=np.float32)).to(torch.bfloat16)
    q, k, v = mk(T, hq, d), mk(T, hkv, d), mk(T, hkv, d)
    kp = torch.zeros(nb, bs, hkv, d, dtype=torch.bfloat16)
    vp = torch.zeros_like(kp)
    max_pos, theta = int(pos.max()) + 1, 500000.0
    table = P.rope_cos_sin_cache(max_pos, d, theta, device=dev)
    q_out, kp_g, vp_g, errbits = _run(dev, q.to(dev), k.to(dev), v.to(dev), kp, vp, slots, pos,
                                      table, True)
    assert errbits == 0
    ref_table = oracle.cos_sin_table(max_pos, d, theta)
    sample = np.sort(rng.choice(T, 96, replace=False))
    qr = oracle.rotate(f64(q[sample]), pos[sample], ref_table, d, True)
    kr = oracle.rotate(f64(k[sample]), pos[sample], ref_table, d, True)
    _close(f64(q_out[sample]), qr, "bf16", "q sample")
    s = slots[sample]
    _close(f64(kp_g)[s // bs, s % bs], kr, "bf16", "k sample")
    assert np.array_equal(bits(vp_g)[slots // bs, slots % bs], bits(v))
    # rotation keeps every head's norm (up to the bf16 rounding of each element)
    n_in = np.linalg.norm(f64(q), axis=-1)
    n_out = np.linalg.norm(f64(q_out), axis=-1)
    assert np.all(np.abs(n_out - n_in) <= 2.0 ** -7 * n_in + 1e-3)

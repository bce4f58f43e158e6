"""FP8 (e4m3) KV cache with per-tensor scales: the cache write stores the
oracle's codes bit for bit, and attention over the e4m3 pools matches the
fp64 oracle over the dequantised pools."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import workloads as W
from _util import assert_close, f64, fp8_codes, oracle_full_fp8

pytestmark = pytest.mark.gpu


def _run(w, dev, out_dtype=torch.float32):
    host = W.make_tensors(w, "cpu", where="host")
    t = {k: v.to(dev) for k, v in host.items()}
    idx = W.index_tensors(w, dev)
    err = P.new_error_word(dev)
    slots = torch.empty(w.num_tokens, dtype=torch.int64, device=dev)
    out = P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
                 idx["query_start_loc"], idx["seq_lens"], w.scale, decode_only=w.is_decode,
                 out_dtype=out_dtype, slots=slots, err=err, kv_scales=w.kv_scales)
    torch.cuda.synchronize()
    return host, t, slots, out, P.read_error(err)


def _check(w, dev):
    host, t, slots, out, errbits = _run(w, dev)
    ref_slots, kc, vc, ref, ref_err, valid = oracle_full_fp8(w, host)
    assert errbits == 0 and ref_err == set()
    assert np.array_equal(slots.cpu().numpy(), ref_slots)
    assert np.array_equal(fp8_codes(t["k_cache"]), kc)          # codes bit for bit
    assert np.array_equal(fp8_codes(t["v_cache"]), vc)
    return assert_close(f64(out)[valid], ref[valid], "bf16", w.name)


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(8, 2), (32, 8), (16, 16)])
def test_fp8_decode(cuda_device, bs, D, hq, hkv):
    rng = np.random.default_rng([bs, D, hq])
    lens = [int(x) for x in rng.integers(1, 900, 7)] + [1, bs, bs + 1]
    w = W.with_fp8_cache(W.custom(f"fp8_dec_{bs}_{D}_{hq}", lens, [1] * len(lens), hq, hkv, D, bs,
                                  "bf16", seed=bs + D + hq, extra_blocks=3))
    _check(w, cuda_device)


@pytest.mark.parametrize("D", [64, 128])
def test_fp8_mixed_step(cuda_device, D):
    lens = [300, 17, 1024, 5, 700]
    qlens = [1, 9, 200, 1, 64]
    w = W.with_fp8_cache(W.custom(f"fp8_mixed_{D}", lens, qlens, 32, 8, D, 16, "bf16", seed=D))
    _check(w, cuda_device)


def test_fp8_every_code_decodes_exactly(cuda_device):
    """One key per request (softmax weight 1): the output is the V row's codes
    times v_scale, for all 254 finite e4m3 codes."""
    dev = cuda_device
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    d, hkv, hq, bs = 128, 2, 2, 16
    n_rows = (len(codes) + d - 1) // d                 # 2 V rows hold every code once
    rows = np.resize(codes, n_rows * d).reshape(n_rows, d)
    nb = n_rows
    kp = np.zeros((nb, bs, hkv, d), dtype=np.uint8)
    vp = np.zeros((nb, bs, hkv, d), dtype=np.uint8)
    for b in range(nb):
        vp[b, 0, :, :] = rows[b]
    scale = 0.0271
    k_cache = torch.from_numpy(kp).view(torch.float8_e4m3fn).to(dev)
    v_cache = torch.from_numpy(vp).view(torch.float8_e4m3fn).to(dev)
    tables = torch.arange(nb, dtype=torch.int32, device=dev).view(nb, 1)
    lens = torch.ones(nb, dtype=torch.int32, device=dev)
    q = torch.randn(nb, hq, d, device=dev).to(torch.bfloat16)
    out = P.decode(q, k_cache, v_cache, tables, lens, 0.1, kv_scales=(0.5, scale)).cpu().numpy()
    want = (oracle.e4m3_decode(rows) * np.float32(scale)).astype(np.float32)
    for b in range(nb):
        for h in range(hq):
            assert np.array_equal(out[b, h], want[b]), (b, h)


def test_fp8_every_key_code_scores_exactly(cuda_device):
    """Two keys per request: key 0 holds one K code in one dim (the dim moves
    with the code, so every k slot of the tensor-core fragments is used), key 1
    is zero, and only key 0's V row is non-zero (1.0 in the same dim).  The
    output there is v_scale * sigmoid(q . k), for all 254 finite e4m3 codes,
    the subnormal ones (zero exponent) included."""
    dev = cuda_device
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    n, d, hkv, hq, bs = len(codes), 128, 2, 8, 16
    vals = oracle.e4m3_decode(codes).astype(np.float64)
    dims = np.arange(n) % d
    kp = np.zeros((n, bs, hkv, d), dtype=np.uint8)
    vp = np.zeros((n, bs, hkv, d), dtype=np.uint8)
    q = np.zeros((n, hq, d), dtype=np.float32)
    heads = (np.arange(hq) - 3.5) * 0.5                  # scores of both signs
    for b in range(n):
        kp[b, 0, :, dims[b]] = codes[b]
        vp[b, 0, :, dims[b]] = 0x38                       # 1.0
        q[b, :, dims[b]] = heads / (vals[b] if vals[b] != 0 else 1.0)
    qb = torch.from_numpy(q).to(torch.bfloat16)
    k_scale, v_scale, sm = 1.0, 0.5, 1.0
    out = P.decode(qb.to(dev), torch.from_numpy(kp).view(torch.float8_e4m3fn).to(dev),
                   torch.from_numpy(vp).view(torch.float8_e4m3fn).to(dev),
                   torch.arange(n, dtype=torch.int32, device=dev).view(n, 1),
                   torch.full((n,), 2, dtype=torch.int32, device=dev), sm,
                   kv_scales=(k_scale, v_scale)).cpu().numpy().astype(np.float64)
    qd = qb.float().numpy().astype(np.float64)
    for b in range(n):
        s0 = qd[b, :, dims[b]] * vals[b] * k_scale * sm
        want = v_scale / (1.0 + np.exp(-s0))
        got = out[b, :, dims[b]]
        assert np.allclose(got, want, rtol=2e-3, atol=1e-6), (hex(codes[b]), got, want)
        rest = np.delete(out[b], dims[b], axis=1)
        assert np.all(rest == 0), hex(codes[b])


def test_fp8_cache_write_saturates_and_skips(cuda_device):
    dev = cuda_device
    T, hkv, d, nb, bs = 6, 2, 64, 4, 8
    scale = 0.01
    k = torch.tensor(np.linspace(-9, 9, T * hkv * d, dtype=np.float32).reshape(T, hkv, d)).to(torch.bfloat16)
    v = -k
    kc = torch.zeros(nb, bs, hkv, d, dtype=torch.float8_e4m3fn, device=dev)
    vc = torch.zeros_like(kc)
    slots = torch.tensor([3, -1, 31, 32, 0, 12], dtype=torch.int64, device=dev)   # 32: past the pool
    err = P.new_error_word(dev)
    P.cache_write(k.to(dev), v.to(dev), kc, vc, slots, err=err, kv_scales=(scale, scale))
    torch.cuda.synchronize()
    assert P.read_error(err) == P.ERRBIT_SLOT_OOB
    kq = oracle.quantize(f64(k).astype(np.float32), scale)
    vq = oracle.quantize(f64(v).astype(np.float32), scale)
    exp_k, exp_v, _ = oracle.cache_write(np.zeros((nb, bs, hkv, d), np.uint8),
                                         np.zeros((nb, bs, hkv, d), np.uint8), kq, vq,
                                         slots.cpu().numpy())
    assert np.array_equal(fp8_codes(kc), exp_k) and np.array_equal(fp8_codes(vc), exp_v)
    assert (fp8_codes(kc) == 0x7E).any() and (fp8_codes(kc) == 0xFE).any()    # saturated

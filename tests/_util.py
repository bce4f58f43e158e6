"""Shared helpers for the GPU parity tests: run the oracle on the same seeded
inputs the CUDA path gets, and compare."""

from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_F32_MAX = 1e-5
TOL_BF16_MAX = 1e-2
TOL_BF16_MEAN = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy()
    return t.numpy()


def oracle_full(w, host):
    """Oracle over a whole (small) workload: slots, cache write, attention.

    host: dict of CPU tensors from workloads.make_tensors.  Returns
    (slots, k_pool_bits, v_pool_bits, out [T,Hq,D] float64, errors, valid).
    """
    qsl = w.query_start_loc
    slots = oracle.slot_mapping(w.block_tables, qsl, w.seq_lens, w.block_size)
    kb, vb, err_w = oracle.cache_write(bits(host["k_cache"]), bits(host["v_cache"]),
                                       bits(host["k_new"]), bits(host["v_new"]), slots)
    k64, v64, _ = oracle.cache_write(f64(host["k_cache"]), f64(host["v_cache"]),
                                     f64(host["k_new"]), f64(host["v_new"]), slots)
    out, err_a, valid = oracle.paged_mixed_step(f64(host["q"]), k64, v64, w.block_tables, qsl,
                                                w.seq_lens, w.scale)
    return slots, kb, vb, out, err_w | err_a, valid


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    if dtype == "f32":
        assert err.max() <= TOL_F32_MAX, f"{what}: max-abs {err.max():.3g} > {TOL_F32_MAX}"
    else:
        assert err.max() <= TOL_BF16_MAX, f"{what}: max-abs {err.max():.3g} > {TOL_BF16_MAX}"
        assert err.mean() <= TOL_BF16_MEAN, f"{what}: mean-abs {err.mean():.3g} > {TOL_BF16_MEAN}"
    return float(err.max()), float(err.mean())


def fp8_codes(t: torch.Tensor) -> np.ndarray:
    """Raw bytes of a float8_e4m3fn tensor."""
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def oracle_full_fp8(w, host):
    """oracle_full for e4m3 pools: the expected pool codes after the cache
    write (oracle quantisation of the new rows) and the attention over the
    dequantised pools.  Returns (slots, k_codes, v_codes, out, errors, valid)."""
    qsl = w.query_start_loc
    slots = oracle.slot_mapping(w.block_tables, qsl, w.seq_lens, w.block_size)
    kc0, vc0 = fp8_codes(host["k_cache"]), fp8_codes(host["v_cache"])
    kq = oracle.quantize(f64(host["k_new"]).astype(np.float32), w.kv_scale)
    vq = oracle.quantize(f64(host["v_new"]).astype(np.float32), w.kv_scale)
    kc, vc, err_w = oracle.cache_write(kc0, vc0, kq, vq, slots)
    k64 = oracle.dequantize(kc, w.kv_scale)
    v64 = oracle.dequantize(vc, w.kv_scale)
    out, err_a, valid = oracle.paged_mixed_step(f64(host["q"]), k64, v64, w.block_tables, qsl,
                                                w.seq_lens, w.scale)
    return slots, kc, vc, out, err_w | err_a, valid


def device_blocks(w, pools, seqs):
    """Device copies of the blocks each request in `seqs` uses, taken before
    the step runs (the oracle applies the step's cache write itself).  Kept on
    the device so that whole outputs of full-size workloads can be checked one
    request at a time without holding every request's history on the host."""
    k_cache, v_cache = pools
    out = {}
    for b in seqs:
        n = (int(w.seq_lens[b]) + w.block_size - 1) // w.block_size
        ids = torch.from_numpy(w.block_tables[b, :n].astype(np.int64)).to(k_cache.device)
        out[int(b)] = (k_cache.index_select(0, ids), v_cache.index_select(0, ids))
    return out


def oracle_request(w, blocks, k_new, v_new, q, b, dequant=None):
    """Oracle output of every query row of request b: [q_b, Hq, D] float64.

    blocks = (k_blocks, v_blocks) of the request as copied before the step
    (pool dtype, any device); k_new / v_new / q are CPU tensors of the step's
    new tokens and queries.  The request's new tokens are written into its
    blocks with the oracle's slot function and cache write, the history is
    gathered through the (renumbered) block table, and all q_b queries attend
    at once.  dequant(codes) turns e4m3 codes into float64 values."""
    qsl = w.query_start_loc
    kb, vb = blocks
    t0, t1 = int(qsl[b]), int(qsl[b + 1])
    q_b, L = t1 - t0, int(w.seq_lens[b])
    n = kb.shape[0]
    table = np.arange(n, dtype=np.int32)[None, :]
    slots = oracle.slot_mapping(table, [0, q_b], [L], w.block_size)
    if dequant is None:
        kk, vv, _ = oracle.cache_write(f64(kb), f64(vb), f64(k_new[t0:t1]), f64(v_new[t0:t1]),
                                       slots)
    else:
        kq = oracle.quantize(f64(k_new[t0:t1]).astype(np.float32), w.kv_scale)
        vq = oracle.quantize(f64(v_new[t0:t1]).astype(np.float32), w.kv_scale)
        kc, vc, _ = oracle.cache_write(fp8_codes(kb), fp8_codes(vb), kq, vq, slots)
        kk, vv = dequant(kc), dequant(vc)
    K = oracle.gather(kk, table[0], L)
    V = oracle.gather(vv, table[0], L)
    return oracle.attend_two_pass(f64(q[t0:t1]), K, V, w.scale, L - q_b)

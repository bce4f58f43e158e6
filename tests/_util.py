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


def oracle_rows(w, host_blocks, k_new, v_new, q, rows):
    """Oracle for selected flattened query rows of a large workload.

    host_blocks[b] = (k_blocks, v_blocks) float64 [n_b, bs, Hkv, D] copied from
    the device pool right after generation (before any kernel ran) for every
    request b that owns a sampled row.  k_new / v_new / q are CPU tensors of the
    step's new tokens and queries.  Returns {row: [Hq, D] float64}.
    """
    qsl = w.query_start_loc
    owner = np.searchsorted(qsl, np.asarray(rows), side="right") - 1
    res = {}
    for r, b in zip(rows, owner):
        b = int(b)
        kb, vb = host_blocks[b]
        n = kb.shape[0]
        table = np.arange(n, dtype=np.int32)[None, :]
        t0, t1 = int(qsl[b]), int(qsl[b + 1])
        q_b, L = t1 - t0, int(w.seq_lens[b])
        slots = oracle.slot_mapping(table, [0, q_b], [L], w.block_size)
        kk, vv, _ = oracle.cache_write(kb, vb, f64(k_new[t0:t1]), f64(v_new[t0:t1]), slots)
        pos = L - q_b + (int(r) - t0)
        K = oracle.gather(kk, table[0], pos + 1)
        V = oracle.gather(vv, table[0], pos + 1)
        res[int(r)] = oracle.attend_two_pass(f64(q[r:r + 1]), K, V, w.scale, pos)[0]
    return res


def snapshot_blocks(w, pools, seqs):
    """Copy the blocks each request in `seqs` uses, as float64 on the host."""
    k_cache, v_cache = pools
    out = {}
    for b in seqs:
        n = (int(w.seq_lens[b]) + w.block_size - 1) // w.block_size
        ids = torch.from_numpy(w.block_tables[b, :n].astype(np.int64)).to(k_cache.device)
        out[int(b)] = (f64(k_cache.index_select(0, ids)), f64(v_cache.index_select(0, ids)))
    return out


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

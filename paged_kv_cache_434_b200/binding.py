"""ctypes binding of libpa_b200.so: argument marshalling only.

Every function takes torch tensors that live on the current CUDA device,
checks dtype / shape / contiguity, and passes raw device pointers, sizes and
the current stream to the C ABI declared in include/pa.h.  All arithmetic
happens in the library's CUDA kernels.  There is no CPU fallback: if the
library cannot be loaded, every call raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libpa_b200.so")

(PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE, PA_ERR_CUDA, PA_ERR_DEVICE_OOB,
 PA_ERR_TIMEOUT) = range(7)
PA_F32, PA_BF16, PA_FP8_E4M3 = 0, 1, 2

ERRBIT_SLOT_OOB = 0x1
ERRBIT_BLOCK_OOB = 0x2
ERRBIT_SEQ_TOO_LONG = 0x4
ERRBIT_QUERY_TOO_LONG = 0x8
ERRBIT_TIMEOUT = 0x10
ERRBIT_POS_OOB = 0x20
ERRBIT_Q_RANGE = 0x40

EXPORTS = ("pa_status_str", "pa_version", "pa_slot_mapping", "pa_cache_write",
           "pa_decode_workspace_size", "pa_decode", "pa_mixed_step_workspace_size",
           "pa_mixed_step", "pa_read_error", "pa_decode_no_alloc", "pa_kernel_timing_enable",
           "pa_kernel_timing_read", "pa_rope_cos_sin_cache", "pa_rope_cache_write",
           "pa_copy_blocks", "pa_slot_mapping_positions", "pa_selftest_wait_timeout",
           "pa_slot_mapping_cache_write", "pa_decode_step")


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib().pa_status_str(status).decode() if _LIB is not None else str(status)
        super().__init__(f"{where}: {msg} (status {status})")


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int64), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("k_scale", ctypes.c_float),
                ("v_scale", ctypes.c_float)]


_LIB = None
_vp, _i32, _i64, _f32, _sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                              ctypes.c_size_t)
_desc_p = ctypes.POINTER(CacheDesc)

_SIGNATURES = {
    "pa_status_str": ([ctypes.c_int], ctypes.c_char_p),
    "pa_version": ([], ctypes.c_int),
    "pa_slot_mapping": ([_vp, _i32, _vp, _vp, _i32, _i64, _i32, _i64, _vp, _vp, _vp], ctypes.c_int),
    "pa_cache_write": ([_vp, _vp, _vp, _vp, _vp, _i64, _desc_p, _vp, _vp], ctypes.c_int),
    "pa_slot_mapping_cache_write": ([_vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _i64, _desc_p,
                                     _vp, _vp, _vp], ctypes.c_int),
    "pa_decode_workspace_size": ([_i32, _i32, _i32, _desc_p], _sz),
    "pa_decode": ([_vp, _vp, _vp, _vp, _vp, _f32, _vp, _i32, _i32, _i32, _i32, _desc_p, _vp, _sz,
                   _vp, _vp], ctypes.c_int),
    "pa_decode_step": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _f32, _vp, _i32, _i32, _i32, _i32,
                        _desc_p, _vp, _vp, _sz, _vp, _vp], ctypes.c_int),
    "pa_mixed_step_workspace_size": ([_i32, _i64, _i32, _i32, _desc_p], _sz),
    "pa_mixed_step": ([_vp, _vp, _vp, _vp, _vp, _vp, _f32, _vp, _i32, _i64, _i32, _i32, _i32,
                       _desc_p, _vp, _sz, _vp, _vp], ctypes.c_int),
    "pa_read_error": ([_vp, ctypes.POINTER(ctypes.c_int32), _vp], ctypes.c_int),
    "pa_decode_no_alloc": ([_vp, _vp, _vp, _vp, _vp, _f32, _vp, _i32, _i32, _i32, _i32, _desc_p,
                            _vp, _vp], ctypes.c_int),
    "pa_kernel_timing_enable": ([_i32], ctypes.c_int),
    "pa_kernel_timing_read": ([ctypes.POINTER(ctypes.c_float)], ctypes.c_int),
    "pa_rope_cos_sin_cache": ([_vp, _i32, _i32, ctypes.c_double, _vp], ctypes.c_int),
    "pa_copy_blocks": ([_vp, _vp, _vp, _i64, _desc_p, _vp, _vp], ctypes.c_int),
    "pa_slot_mapping_positions": ([_vp, _i32, _i32, _vp, _vp, _i64, _i32, _i64, _vp, _vp, _vp],
                                  ctypes.c_int),
    "pa_selftest_wait_timeout": ([ctypes.c_uint32, _vp, _vp, _vp], ctypes.c_int),
    "pa_rope_cache_write": ([_vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32,
                             _i32, _i64, _i32, _desc_p, _vp, _vp], ctypes.c_int),
}

# Launch kinds timed by kernel_timing (PA_TK_* order).
TIMED_KERNELS = ("plan", "tiles", "decode", "merge")

# Size of the library's static scratch used by decode_no_alloc (PA_DECODE_NO_ALLOC_MAX_BYTES).
DECODE_NO_ALLOC_MAX_BYTES = 32 << 20


def library_path() -> str:
    return _LIB_PATH


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"libpa_b200.so not found at {_LIB_PATH}; build it with "
                "`python -m paged_kv_cache_434_b200.build` (needs nvcc, sm_100a)")
        lib = ctypes.CDLL(_LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = lib
    return _LIB


def version() -> int:
    return _lib().pa_version()


# ---------------------------------------------------------------- helpers

def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return PA_F32
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.float8_e4m3fn:
        return PA_FP8_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}; use float32, bfloat16 or float8_e4m3fn pools")


def _cuda(t: torch.Tensor, name: str, dtype=None, ndim=None) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    return t.data_ptr()


def _entries(t, name: str, count: int, ndim: int = 1):
    """The library reads `count` rows of `t` through a raw pointer: refuse a
    tensor with fewer, which would be read past its end on the device."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dim() != ndim or t.shape[0] < count:
        raise ValueError(f"{name} must be a {ndim}-D tensor with at least {count} rows, "
                         f"got shape {tuple(t.shape)}")


def _out_shape(out, shape):
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"out must have shape {tuple(shape)}, got {tuple(out.shape)}")


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _err_ptr(err):
    if err is None:
        return None
    return _cuda(err, "err", torch.int32)


def cache_desc(k_cache: torch.Tensor, kv_scales=None) -> CacheDesc:
    """Descriptor of a layer's pools.  float8_e4m3fn pools need kv_scales =
    (k_scale, v_scale): an entry stands for code * scale."""
    nb, bs, hkv, d = k_cache.shape
    dt = _dt(k_cache)
    ks = vs = 1.0
    if dt == PA_FP8_E4M3:
        if kv_scales is None:
            raise ValueError("float8_e4m3fn pools need kv_scales=(k_scale, v_scale)")
        ks, vs = (float(x) for x in kv_scales)
    return CacheDesc(nb, bs, hkv, d, dt, ks, vs)


def io_dtype(k_cache: torch.Tensor):
    """dtype of the queries and new K/V rows that go with these pools."""
    return torch.bfloat16 if k_cache.dtype == torch.float8_e4m3fn else k_cache.dtype


def _any_scales(k_cache):
    return (1.0, 1.0) if k_cache.dtype == torch.float8_e4m3fn else None


def _check(status: int, where: str):
    if status != PA_OK:
        raise PagedAttentionError(status, where)


def new_error_word(device=None) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def read_error(err: torch.Tensor) -> int:
    """Synchronise the current stream, return the error bits and clear them."""
    bits = ctypes.c_int32(0)
    st = _lib().pa_read_error(_cuda(err, "err", torch.int32), ctypes.byref(bits), _stream())
    if st not in (PA_OK, PA_ERR_DEVICE_OOB, PA_ERR_TIMEOUT):
        raise PagedAttentionError(st, "pa_read_error")
    return bits.value


def kernel_timing(enable: bool) -> None:
    """Turn per-launch event timing of attention calls on or off (current device)."""
    _check(_lib().pa_kernel_timing_enable(1 if enable else 0), "pa_kernel_timing_enable")


def kernel_times() -> dict:
    """Device ms of each launch of the last timed attention call (absent: not launched)."""
    ms = (ctypes.c_float * len(TIMED_KERNELS))()
    _check(_lib().pa_kernel_timing_read(ms), "pa_kernel_timing_read")
    return {k: float(v) for k, v in zip(TIMED_KERNELS, ms) if v >= 0}


# ---------------------------------------------------------------- operations

def slot_mapping(block_tables, query_start_loc, seq_lens, block_size: int, num_blocks: int,
                 num_tokens: int, out=None, err=None):
    """int64 slot of every new token (see pa_slot_mapping)."""
    B, W = block_tables.shape
    _entries(query_start_loc, "query_start_loc", B + 1)
    _entries(seq_lens, "seq_lens", B)
    if out is None:
        out = torch.empty(num_tokens, dtype=torch.int64, device=block_tables.device)
    _entries(out, "slot_mapping", num_tokens)
    _check(_lib().pa_slot_mapping(
        _cuda(block_tables, "block_tables", torch.int32, 2), W,
        _cuda(query_start_loc, "query_start_loc", torch.int32, 1),
        _cuda(seq_lens, "seq_lens", torch.int32, 1), B, num_tokens, block_size, num_blocks,
        _cuda(out, "slot_mapping", torch.int64, 1), _err_ptr(err), _stream()), "pa_slot_mapping")
    return out


def cache_write(k, v, k_cache, v_cache, slot_mapping, err=None, kv_scales=None):
    """reshape_and_cache: k_cache[slot // bs, slot % bs] = k[t] (and v); FP8
    pools store the e4m3 code of k / k_scale (and v / v_scale)."""
    desc = cache_desc(k_cache, kv_scales)
    T = k.shape[0]
    for name, t in (("k", k), ("v", v)):
        if t.dim() != 3 or tuple(t.shape[1:]) != (desc.num_kv_heads, desc.head_dim) or \
                t.shape[0] != T or t.dtype != io_dtype(k_cache):
            raise ValueError(f"{name} must be [num_tokens, num_kv_heads, head_dim] of the cache's "
                             f"input dtype")
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise ValueError("v_cache must match k_cache")
    if slot_mapping.shape[0] != T:
        raise ValueError("slot_mapping must have num_tokens entries")
    _check(_lib().pa_cache_write(
        _cuda(k, "k"), _cuda(v, "v"), _cuda(k_cache, "k_cache", ndim=4),
        _cuda(v_cache, "v_cache", ndim=4), _cuda(slot_mapping, "slot_mapping", torch.int64, 1),
        T, ctypes.byref(desc), _err_ptr(err), _stream()), "pa_cache_write")


def slot_mapping_cache_write(k, v, k_cache, v_cache, block_tables, query_start_loc, seq_lens,
                             slots=None, err=None, kv_scales=None):
    """slot_mapping then cache_write in one launch (see pa_slot_mapping_cache_write).
    query_start_loc None: a decode step, one new token per request.  Returns
    the slots (allocated unless `slots` is given)."""
    desc = cache_desc(k_cache, kv_scales)
    T = k.shape[0]
    B, W = block_tables.shape
    for name, t in (("k", k), ("v", v)):
        if t.dim() != 3 or tuple(t.shape[1:]) != (desc.num_kv_heads, desc.head_dim) or \
                t.shape[0] != T or t.dtype != io_dtype(k_cache):
            raise ValueError(f"{name} must be [num_tokens, num_kv_heads, head_dim] of the cache's "
                             f"input dtype")
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise ValueError("v_cache must match k_cache")
    _entries(seq_lens, "seq_lens", B)
    if query_start_loc is not None:
        _entries(query_start_loc, "query_start_loc", B + 1)
    elif T != B:
        raise ValueError("without query_start_loc every request has exactly one new token")
    if slots is None:
        slots = torch.empty(T, dtype=torch.int64, device=k.device)
    _entries(slots, "slot_mapping", T)
    _check(_lib().pa_slot_mapping_cache_write(
        _cuda(k, "k"), _cuda(v, "v"), _cuda(k_cache, "k_cache", ndim=4),
        _cuda(v_cache, "v_cache", ndim=4), _cuda(block_tables, "block_tables", torch.int32, 2), W,
        None if query_start_loc is None else _cuda(query_start_loc, "query_start_loc", torch.int32, 1),
        _cuda(seq_lens, "seq_lens", torch.int32, 1), B, T, ctypes.byref(desc),
        _cuda(slots, "slot_mapping", torch.int64, 1), _err_ptr(err), _stream()),
        "pa_slot_mapping_cache_write")
    return slots


def copy_blocks(k_cache, v_cache, block_mapping, err=None):
    """Copy-on-write block copies: block dst := block src in both pools for
    every (src, dst) row of the int64 [num_pairs, 2] block_mapping."""
    desc = cache_desc(k_cache, _any_scales(k_cache))
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise ValueError("v_cache must match k_cache")
    if block_mapping.dim() != 2 or block_mapping.shape[1] != 2:
        raise ValueError("block_mapping must be [num_pairs, 2]")
    _check(_lib().pa_copy_blocks(
        _cuda(k_cache, "k_cache", ndim=4), _cuda(v_cache, "v_cache", ndim=4),
        _cuda(block_mapping, "block_mapping", torch.int64, 2), block_mapping.shape[0],
        ctypes.byref(desc), _err_ptr(err), _stream()), "pa_copy_blocks")


def slot_mapping_positions(block_tables, token_req, positions, block_size: int, num_blocks: int,
                           out=None, err=None):
    """int64 slot of every token from its request index and position."""
    B, W = block_tables.shape
    T = positions.shape[0]
    if token_req.shape[0] != T:
        raise ValueError("token_req and positions must have one entry per token")
    if out is None:
        out = torch.empty(T, dtype=torch.int64, device=positions.device)
    _entries(out, "out", T)
    _check(_lib().pa_slot_mapping_positions(
        _cuda(block_tables, "block_tables", torch.int32, 2), W, B,
        _cuda(token_req, "token_req", torch.int32, 1), _cuda(positions, "positions", torch.int64, 1),
        T, block_size, num_blocks, _cuda(out, "out", torch.int64, 1), _err_ptr(err), _stream()),
        "pa_slot_mapping_positions")
    return out


def rope_cos_sin_cache(max_position: int, rotary_dim: int, theta: float, device=None,
                       out=None) -> torch.Tensor:
    """float32 [max_position, rotary_dim] rotary table (see pa_rope_cos_sin_cache)."""
    if out is None:
        out = torch.empty(max_position, rotary_dim, dtype=torch.float32,
                          device=device or "cuda")
    if tuple(out.shape) != (max_position, rotary_dim):
        raise ValueError("out must be [max_position, rotary_dim]")
    _check(_lib().pa_rope_cos_sin_cache(_cuda(out, "out", torch.float32, 2), max_position,
                                        rotary_dim, float(theta), _stream()),
           "pa_rope_cos_sin_cache")
    return out


def _token_rows(t: torch.Tensor, name: str, heads: int, d: int) -> int:
    """Token stride (elements) of a [T, heads, d] view whose heads of one token
    are contiguous (a column slice of a fused QKV output qualifies)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 3 or tuple(t.shape[1:]) != (heads, d) or t.stride(2) != 1 or t.stride(1) != d:
        raise ValueError(f"{name} must be a [num_tokens, {heads}, {d}] view with contiguous heads")
    return t.stride(0)


def rope_cache_write(q, k, v, k_cache, v_cache, slot_mapping, positions, cos_sin_cache,
                     neox: bool = True, q_out=None, err=None):
    """Rotate q and k by their positions, store rotated k and plain v at their
    slots, return the rotated queries (see pa_rope_cache_write)."""
    desc = cache_desc(k_cache, _any_scales(k_cache))
    T, Hq, D = q.shape
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise ValueError("v_cache must match k_cache")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != k_cache.dtype or t.shape[0] != T:
            raise ValueError(f"{name} must have num_tokens rows of the cache dtype")
    _entries(slot_mapping, "slot_mapping", T)
    _entries(positions, "positions", T)
    qs = _token_rows(q, "q", Hq, D)
    ks = _token_rows(k, "k", desc.num_kv_heads, desc.head_dim)
    if _token_rows(v, "v", desc.num_kv_heads, desc.head_dim) != ks:
        raise ValueError("k and v must share their token stride")
    if q_out is None:
        q_out = torch.empty(T, Hq, D, dtype=q.dtype, device=q.device)
    if not q_out.is_contiguous() or tuple(q_out.shape) != (T, Hq, D) or q_out.dtype != q.dtype:
        raise ValueError("q_out must be a contiguous [num_tokens, num_heads, head_dim] tensor")
    max_pos, rot = cos_sin_cache.shape
    _check(_lib().pa_rope_cache_write(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), qs, ks, q_out.data_ptr(),
        _cuda(k_cache, "k_cache", ndim=4), _cuda(v_cache, "v_cache", ndim=4),
        _cuda(positions, "positions", torch.int64, 1),
        _cuda(slot_mapping, "slot_mapping", torch.int64, 1),
        _cuda(cos_sin_cache, "cos_sin_cache", torch.float32, 2), max_pos, rot, 1 if neox else 0,
        T, Hq, ctypes.byref(desc), _err_ptr(err), _stream()), "pa_rope_cache_write")
    return q_out


def decode_workspace_size(num_seqs, num_heads, max_blocks_per_seq, k_cache) -> int:
    desc = cache_desc(k_cache, _any_scales(k_cache))
    return int(_lib().pa_decode_workspace_size(num_seqs, num_heads, max_blocks_per_seq,
                                               ctypes.byref(desc)))


def mixed_step_workspace_size(num_seqs, num_tokens, num_heads, max_blocks_per_seq, k_cache) -> int:
    desc = cache_desc(k_cache, _any_scales(k_cache))
    return int(_lib().pa_mixed_step_workspace_size(num_seqs, num_tokens, num_heads,
                                                   max_blocks_per_seq, ctypes.byref(desc)))


def _workspace(nbytes, device, workspace):
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _check_attn(q, k_cache, v_cache, block_tables, seq_lens, out_dtype, kv_scales=None,
                num_seqs=None):
    desc = cache_desc(k_cache, kv_scales)
    if num_seqs is not None:
        _entries(block_tables, "block_tables", num_seqs, ndim=2)
        _entries(seq_lens, "seq_lens", num_seqs)
    if q.dtype != io_dtype(k_cache) or q.dim() != 3 or q.shape[2] != desc.head_dim:
        raise ValueError("q must be [rows, num_heads, head_dim] of the cache's input dtype")
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise ValueError("v_cache must match k_cache")
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out_dtype must be float32 or bfloat16")
    return desc


def decode(q, k_cache, v_cache, block_tables, seq_lens, scale: float, out=None,
           out_dtype=torch.float32, workspace=None, err=None, kv_scales=None):
    """Decode attention: out[b, h] over the first seq_lens[b] keys of request b."""
    desc = _check_attn(q, k_cache, v_cache, block_tables, seq_lens, out_dtype, kv_scales,
                       num_seqs=q.shape[0] if q.dim() == 3 else None)
    B, H, D = q.shape
    W = block_tables.shape[1]
    if out is None:
        out = torch.empty(B, H, D, dtype=out_dtype, device=q.device)
    _out_shape(out, (B, H, D))
    nbytes = decode_workspace_size(B, H, W, k_cache)
    ws = _workspace(nbytes, q.device, workspace)
    _check(_lib().pa_decode(
        _cuda(q, "q"), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
        _cuda(block_tables, "block_tables", torch.int32, 2),
        _cuda(seq_lens, "seq_lens", torch.int32, 1), float(scale), _cuda(out, "out"), B, H, W,
        _dt(out), ctypes.byref(desc), _cuda(ws, "workspace"), ws.numel() * ws.element_size(),
        _err_ptr(err), _stream()), "pa_decode")
    return out


def decode_step(q, k, v, k_cache, v_cache, block_tables, seq_lens, scale: float, out=None,
                out_dtype=torch.float32, slots=None, workspace=None, err=None, kv_scales=None):
    """One decode step: the new K/V rows (token b of request b) go to their
    slots, then decode attention -- slot_mapping_cache_write(..., None, ...)
    followed by decode(...), the write done in the planner's launch.  Returns
    (out, slots)."""
    desc = _check_attn(q, k_cache, v_cache, block_tables, seq_lens, out_dtype, kv_scales,
                       num_seqs=q.shape[0] if q.dim() == 3 else None)
    B, H, D = q.shape
    W = block_tables.shape[1]
    for name, t in (("k", k), ("v", v)):
        if t.dim() != 3 or tuple(t.shape) != (B, desc.num_kv_heads, desc.head_dim) or \
                t.dtype != io_dtype(k_cache):
            raise ValueError(f"{name} must be [num_seqs, num_kv_heads, head_dim] of the cache's "
                             f"input dtype")
    if out is None:
        out = torch.empty(B, H, D, dtype=out_dtype, device=q.device)
    _out_shape(out, (B, H, D))
    if slots is None:
        slots = torch.empty(B, dtype=torch.int64, device=q.device)
    _entries(slots, "slot_mapping", B)
    nbytes = decode_workspace_size(B, H, W, k_cache)
    ws = _workspace(nbytes, q.device, workspace)
    _check(_lib().pa_decode_step(
        _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"), _cuda(k_cache, "k_cache"),
        _cuda(v_cache, "v_cache"), _cuda(block_tables, "block_tables", torch.int32, 2),
        _cuda(seq_lens, "seq_lens", torch.int32, 1), float(scale), _cuda(out, "out"), B, H, W,
        _dt(out), ctypes.byref(desc), _cuda(slots, "slot_mapping", torch.int64, 1),
        _cuda(ws, "workspace"), ws.numel() * ws.element_size(), _err_ptr(err), _stream()),
        "pa_decode_step")
    return out, slots


def mixed_step(q, k_cache, v_cache, block_tables, query_start_loc, seq_lens, scale: float,
               out=None, out_dtype=torch.float32, workspace=None, err=None, kv_scales=None):
    """Causal varlen attention of a flattened step (chunked prefill + decode)."""
    desc = _check_attn(q, k_cache, v_cache, block_tables, seq_lens, out_dtype, kv_scales,
                       num_seqs=block_tables.shape[0] if block_tables.dim() == 2 else None)
    T, H, D = q.shape
    B, W = block_tables.shape
    _entries(query_start_loc, "query_start_loc", B + 1)
    if out is None:
        out = torch.empty(T, H, D, dtype=out_dtype, device=q.device)
    _out_shape(out, (T, H, D))
    nbytes = mixed_step_workspace_size(B, T, H, W, k_cache)
    ws = _workspace(nbytes, q.device, workspace)
    _check(_lib().pa_mixed_step(
        _cuda(q, "q"), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
        _cuda(block_tables, "block_tables", torch.int32, 2),
        _cuda(query_start_loc, "query_start_loc", torch.int32, 1),
        _cuda(seq_lens, "seq_lens", torch.int32, 1), float(scale), _cuda(out, "out"), B, T, H, W,
        _dt(out), ctypes.byref(desc), _cuda(ws, "workspace"), ws.numel() * ws.element_size(),
        _err_ptr(err), _stream()), "pa_mixed_step")
    return out


def decode_no_alloc(q, k_cache, v_cache, block_tables, seq_lens, scale: float, out,
                    err=None, kv_scales=None):
    """pa_decode_no_alloc: decode attention for callers that can't allocate
    device memory (e.g. a plug-in inside an engine that owns all allocations).

    Same arguments and results as decode(), except that there is no workspace:
    the library uses its own static device scratch of DECODE_NO_ALLOC_MAX_BYTES
    and rejects larger problems with PagedAttentionError (PA_ERR_WORKSPACE).
    `out` must be given, so that this call allocates nothing either.  Calls
    whose kernels overlap on the GPU share the scratch and race.
    """
    desc = _check_attn(q, k_cache, v_cache, block_tables, seq_lens, out.dtype, kv_scales,
                       num_seqs=q.shape[0] if q.dim() == 3 else None)
    B, H, D = q.shape
    W = block_tables.shape[1]
    _out_shape(out, (B, H, D))
    _check(_lib().pa_decode_no_alloc(
        _cuda(q, "q"), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
        _cuda(block_tables, "block_tables", torch.int32, 2),
        _cuda(seq_lens, "seq_lens", torch.int32, 1), float(scale), _cuda(out, "out"), B, H, W,
        _dt(out), ctypes.byref(desc), _err_ptr(err), _stream()), "pa_decode_no_alloc")
    return out


def selftest_wait_timeout(limit_us: int, err, waited_ns=None) -> None:
    """pa_selftest_wait_timeout: one warp waits, through the kernels' bounded
    wait, on an mbarrier nothing arrives at.  The wait must give up after
    `limit_us` microseconds (1 .. 100000) and OR PA_ERRBIT_TIMEOUT into `err`.
    `waited_ns` (an int64 CUDA tensor of one element, or None) receives the
    wait's duration by the GPU's global timer.  Asynchronous on the current
    stream."""
    ptr = None
    if waited_ns is not None:
        ptr = _cuda(waited_ns, "waited_ns", torch.int64)
    _check(_lib().pa_selftest_wait_timeout(int(limit_us), _err_ptr(err), ptr, _stream()),
           "pa_selftest_wait_timeout")

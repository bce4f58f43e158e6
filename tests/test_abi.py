"""The C-ABI library loads and exports what include/pa.h declares; host-side
argument validation returns status codes without touching a GPU."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_434_b200 import binding
    if not os.path.exists(binding.library_path()):
        from paged_kv_cache_434_b200 import build
        build.build()
    return binding._lib()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("pa_cache_write", "pa_decode", "pa_mixed_step", "pa_slot_mapping",
              "pa_read_error", "pa_decode_workspace_size", "pa_mixed_step_workspace_size",
              "pa_status_str", "pa_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(os.path.join(ROOT, "paged_kv_cache_434_b200", "lib", "libpa_b200.so"))
    missing = [n for n in _declared() if not hasattr(raw, n)]
    assert not missing, missing


def test_binding_covers_every_export():
    from paged_kv_cache_434_b200 import binding
    assert sorted(binding.EXPORTS) == sorted(_declared())


def test_status_strings(lib):
    for s in range(7):
        assert lib.pa_status_str(s) and lib.pa_status_str(s) != b"unknown status", s
    assert lib.pa_status_str(99) == b"unknown status"
    assert lib.pa_version() >= 100


def _desc(**kw):
    from paged_kv_cache_434_b200.binding import CacheDesc
    d = dict(num_blocks=16, block_size=16, num_kv_heads=2, head_dim=64, dtype=0)
    d.update(kw)
    return CacheDesc(**d)


def test_cache_write_validation(lib):
    from paged_kv_cache_434_b200 import binding as B
    d = _desc()
    # null pointers
    assert lib.pa_cache_write(None, None, None, None, None, 4, ctypes.byref(d), None, None) == \
        B.PA_ERR_INVALID_ARG
    # zero tokens is a no-op
    assert lib.pa_cache_write(None, None, None, None, None, 0, ctypes.byref(d), None, None) == B.PA_OK
    # unsupported geometry
    for bad in (dict(head_dim=96), dict(block_size=12), dict(dtype=7)):
        assert lib.pa_cache_write(None, None, None, None, None, 1, ctypes.byref(_desc(**bad)),
                                  None, None) == B.PA_ERR_UNSUPPORTED
    assert lib.pa_cache_write(None, None, None, None, None, 1, None, None, None) == \
        B.PA_ERR_INVALID_ARG
    # misaligned device pointer (never dereferenced: rejected on the host)
    assert lib.pa_cache_write(8, 16, 16, 16, 16, 1, ctypes.byref(d), None, None) == \
        B.PA_ERR_INVALID_ARG


def test_attention_validation(lib):
    from paged_kv_cache_434_b200 import binding as B
    d = _desc()
    # num_heads not a multiple of num_kv_heads
    assert lib.pa_decode(16, 16, 16, 16, 16, 0.1, 16, 2, 3, 4, 0, ctypes.byref(d), 256, 1 << 20,
                         None, None) == B.PA_ERR_INVALID_ARG
    # group larger than 16 query heads per KV head
    assert lib.pa_decode(16, 16, 16, 16, 16, 0.1, 16, 2, 64, 4, 0, ctypes.byref(d), 256, 1 << 20,
                         None, None) == B.PA_ERR_UNSUPPORTED
    # bad out dtype
    assert lib.pa_decode(16, 16, 16, 16, 16, 0.1, 16, 2, 8, 4, 5, ctypes.byref(d), 256, 1 << 20,
                         None, None) == B.PA_ERR_UNSUPPORTED
    # null tensors
    assert lib.pa_decode(None, 16, 16, 16, 16, 0.1, 16, 2, 8, 4, 0, ctypes.byref(d), 256,
                         1 << 20, None, None) == B.PA_ERR_INVALID_ARG
    # workspace too small / missing / misaligned
    assert lib.pa_decode(16, 16, 16, 16, 16, 0.1, 16, 2, 8, 4, 0, ctypes.byref(d), 256, 16,
                         None, None) == B.PA_ERR_WORKSPACE
    assert lib.pa_decode(16, 16, 16, 16, 16, 0.1, 16, 2, 8, 4, 0, ctypes.byref(d), None,
                         1 << 20, None, None) == B.PA_ERR_WORKSPACE
    assert lib.pa_decode(16, 16, 16, 16, 16, 0.1, 16, 2, 8, 4, 0, ctypes.byref(d), 272,
                         1 << 20, None, None) == B.PA_ERR_WORKSPACE
    assert lib.pa_mixed_step(16, 16, 16, 16, None, 16, 0.1, 16, 2, 5, 8, 4, 0, ctypes.byref(d),
                             256, 1 << 20, None, None) == B.PA_ERR_INVALID_ARG
    # zero requests is a no-op
    assert lib.pa_decode(None, None, None, None, None, 0.1, None, 0, 8, 4, 0, ctypes.byref(d),
                         None, 0, None, None) == B.PA_OK


def test_decode_step_validation(lib):
    """pa_decode_step refuses what pa_decode refuses, and a NULL or misaligned
    new K/V row buffer, before launching anything."""
    from paged_kv_cache_434_b200 import binding as B
    d = _desc()

    def call(q=16, k=16, v=16, heads=8, out_dtype=0, ws=256, ws_bytes=1 << 20, num_seqs=2):
        return lib.pa_decode_step(q, k, v, 16, 16, 16, 16, 0.1, 16, num_seqs, heads, 4, out_dtype,
                                  ctypes.byref(d), None, ws, ws_bytes, None, None)

    assert call(k=None) == B.PA_ERR_INVALID_ARG
    assert call(v=None) == B.PA_ERR_INVALID_ARG
    assert call(v=24) == B.PA_ERR_INVALID_ARG            # not 16-byte aligned
    assert call(q=None) == B.PA_ERR_INVALID_ARG
    assert call(heads=3) == B.PA_ERR_INVALID_ARG         # not a multiple of num_kv_heads
    assert call(heads=64) == B.PA_ERR_UNSUPPORTED        # group above 16
    assert call(out_dtype=5) == B.PA_ERR_UNSUPPORTED
    assert call(ws_bytes=16) == B.PA_ERR_WORKSPACE
    assert call(ws=None) == B.PA_ERR_WORKSPACE
    assert call(ws=272) == B.PA_ERR_WORKSPACE            # not 256-byte aligned
    assert call(q=None, k=None, v=None, num_seqs=0) == B.PA_OK


def test_workspace_sizes_are_positive_and_monotone(lib):
    d = _desc(num_kv_heads=8, head_dim=128, dtype=1)
    a = lib.pa_decode_workspace_size(64, 32, 512, ctypes.byref(d))
    b = lib.pa_decode_workspace_size(128, 32, 512, ctypes.byref(d))
    assert 0 < a <= b
    assert lib.pa_decode_workspace_size(64, 33, 512, ctypes.byref(d)) == 0
    m = lib.pa_mixed_step_workspace_size(4098, 8192, 32, 384, ctypes.byref(d))
    assert m > 0


def test_workspace_beyond_any_device_is_refused(lib):
    """Arguments whose exact workspace would not fit a size_t (2^26 KV heads,
    2^30 requests) get size 0 and PA_ERR_UNSUPPORTED, never a wrapped size."""
    from paged_kv_cache_434_b200 import binding as B
    for hkv, seqs in ((1 << 26, 1 << 30), (1 << 29, 1 << 30), (1 << 30, 1 << 20)):
        d = _desc(num_blocks=1 << 20, num_kv_heads=hkv, head_dim=128, dtype=1)
        assert lib.pa_decode_workspace_size(seqs, hkv, 4, ctypes.byref(d)) == 0
        assert lib.pa_mixed_step_workspace_size(seqs, seqs, hkv, 4, ctypes.byref(d)) == 0
        assert lib.pa_decode(16, 16, 16, 16, 16, 0.1, 16, seqs, hkv, 4, 0, ctypes.byref(d), 256,
                             1 << 62, None, None) == B.PA_ERR_UNSUPPORTED
        assert lib.pa_mixed_step(16, 16, 16, 16, 16, 16, 0.1, 16, seqs, seqs, hkv, 4, 0,
                                 ctypes.byref(d), 256, 1 << 62, None, None) == \
            B.PA_ERR_UNSUPPORTED


def test_slot_mapping_validation(lib):
    from paged_kv_cache_434_b200 import binding as B
    assert lib.pa_slot_mapping(None, 3, None, None, 2, 5, 16, 16, None, None, None) == \
        B.PA_ERR_INVALID_ARG
    assert lib.pa_slot_mapping(None, 3, None, None, 0, 0, 16, 16, None, None, None) == B.PA_OK
    assert lib.pa_slot_mapping(16, 3, 16, 16, 2, 5, 0, 16, 16, None, None) == B.PA_ERR_INVALID_ARG


def test_product_path_has_no_cpu_fallback():
    """Calls on CPU tensors raise instead of computing anything on the host."""
    import torch
    import paged_kv_cache_434_b200 as P
    kc = torch.zeros(4, 16, 2, 64)
    with pytest.raises(ValueError):
        P.decode(torch.zeros(1, 8, 64), kc, kc, torch.zeros(1, 1, dtype=torch.int32),
                 torch.ones(1, dtype=torch.int32), 0.1)


def test_product_code_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "paged_kv_cache_434_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_kernel_timing_off_paths(lib):
    from paged_kv_cache_434_b200 import binding as B
    ms = (ctypes.c_float * 4)()
    assert lib.pa_kernel_timing_enable(0) == B.PA_OK          # off while off: no CUDA call
    assert lib.pa_kernel_timing_read(ms) == B.PA_ERR_INVALID_ARG
    assert lib.pa_kernel_timing_read(None) == B.PA_ERR_INVALID_ARG


def test_fp8_descriptor_validation(lib):
    from paged_kv_cache_434_b200 import binding as B
    ok = _desc(dtype=2, k_scale=0.5, v_scale=0.25)
    # zero tokens: nothing to do once the descriptor is valid
    assert lib.pa_cache_write(None, None, None, None, None, 0, ctypes.byref(ok), None, None) == B.PA_OK
    for bad in (dict(k_scale=0.0, v_scale=1.0), dict(k_scale=1.0, v_scale=-2.0),
                dict(k_scale=float("inf"), v_scale=1.0), dict(k_scale=float("nan"), v_scale=1.0)):
        d = _desc(dtype=2, **bad)
        assert lib.pa_cache_write(None, None, None, None, None, 0, ctypes.byref(d), None,
                                  None) == B.PA_ERR_INVALID_ARG
    # rotary embedding does not take an e4m3 cache
    assert lib.pa_rope_cache_write(16, 16, 16, 512, 128, 32, 16, 16, 16, 16, 16, 64, 64, 1, 1, 4,
                                   ctypes.byref(ok), None, None) == B.PA_ERR_UNSUPPORTED


def test_rope_validation(lib):
    from paged_kv_cache_434_b200 import binding as B
    d = _desc(head_dim=64)
    call = lambda **kw: lib.pa_rope_cache_write(  # noqa: E731
        kw.get("q", 16), 16, 16, kw.get("qs", 4 * 64), kw.get("ks", 2 * 64), kw.get("qo", 1 << 20),
        16, 16, 16, 16, 16, 64, kw.get("rot", 64), 1, kw.get("T", 3), 4, ctypes.byref(d), None,
        None)
    assert call(rot=24) == B.PA_ERR_UNSUPPORTED               # not a multiple of 16
    assert call(rot=128) == B.PA_ERR_UNSUPPORTED              # larger than head_dim
    assert call(qs=64) == B.PA_ERR_INVALID_ARG                # q rows shorter than 4 heads
    assert call(ks=36) == B.PA_ERR_INVALID_ARG                # not a multiple of 8 elements
    assert call(qo=16 + 64) == B.PA_ERR_INVALID_ARG           # q_out overlaps q_in, not equal
    assert call(q=None) == B.PA_ERR_INVALID_ARG
    assert call(T=0, q=None) == B.PA_OK                       # nothing to do
    assert lib.pa_rope_cos_sin_cache(None, 16, 16, 1e4, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_rope_cos_sin_cache(16, 16, 15, 1e4, None) == B.PA_ERR_INVALID_ARG   # odd
    assert lib.pa_rope_cos_sin_cache(16, 16, 16, 0.0, None) == B.PA_ERR_INVALID_ARG


def test_block_management_validation(lib):
    from paged_kv_cache_434_b200 import binding as B
    d = _desc()
    assert lib.pa_copy_blocks(16, 16, 16, -1, ctypes.byref(d), None, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(None, None, None, 0, ctypes.byref(d), None, None) == B.PA_OK
    assert lib.pa_copy_blocks(None, 16, 16, 3, ctypes.byref(d), None, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(8, 16, 16, 3, ctypes.byref(d), None, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_slot_mapping_positions(None, 4, 2, None, None, 5, 16, 16, None, None, None) == \
        B.PA_ERR_INVALID_ARG
    assert lib.pa_slot_mapping_positions(None, 4, 2, None, None, 0, 16, 16, None, None, None) == \
        B.PA_OK
    assert lib.pa_slot_mapping_positions(16, 4, 2, 16, 16, 5, 0, 16, 16, None, None) == \
        B.PA_ERR_INVALID_ARG                                 # block size 0


def test_binding_refuses_arrays_the_library_would_overrun():
    """The library reads num_seqs rows of block_tables / seq_lens (num_seqs + 1
    of query_start_loc) and writes exactly [rows, Hq, D] through raw pointers:
    the binding refuses shorter arrays and mis-shaped outputs before any call
    (CPU tensors here, so nothing reaches a device)."""
    import torch
    import paged_kv_cache_434_b200 as P
    from paged_kv_cache_434_b200 import binding as B
    kc = torch.zeros(4, 16, 2, 64)
    q = torch.zeros(2, 8, 64)
    kv = torch.zeros(2, 2, 64)
    i32 = lambda *s: torch.zeros(*s, dtype=torch.int32)  # noqa: E731
    cases = [
        (lambda: P.decode(q, kc, kc, i32(1, 3), i32(2), 0.1), "block_tables"),
        (lambda: P.decode(q, kc, kc, i32(2, 3), i32(1), 0.1), "seq_lens"),
        (lambda: P.decode(q, kc, kc, i32(2, 3), i32(2), 0.1, out=torch.zeros(2, 8, 32)), "out"),
        (lambda: P.mixed_step(q, kc, kc, i32(2, 3), i32(2), i32(2), 0.1), "query_start_loc"),
        (lambda: P.mixed_step(q, kc, kc, i32(2, 3), i32(3), i32(1), 0.1), "seq_lens"),
        (lambda: P.mixed_step(q, kc, kc, i32(2, 3), i32(3), i32(2), 0.1,
                              out=torch.zeros(1, 8, 64)), "out"),
        (lambda: B.decode_no_alloc(q, kc, kc, i32(2, 3), i32(2), 0.1, torch.zeros(3, 8, 64)),
         "out"),
        (lambda: P.decode_step(q, kv, kv, kc, kc, i32(1, 3), i32(2), 0.1), "block_tables"),
        (lambda: P.decode_step(q, kv, kv, kc, kc, i32(2, 3), i32(1), 0.1), "seq_lens"),
        (lambda: P.decode_step(q, kv, kv, kc, kc, i32(2, 3), i32(2), 0.1,
                               out=torch.zeros(2, 8, 32)), "out"),
        (lambda: P.decode_step(q, kv, kv, kc, kc, i32(2, 3), i32(2), 0.1,
                               slots=torch.zeros(1, dtype=torch.int64)), "slot_mapping"),
        (lambda: P.slot_mapping(i32(2, 3), i32(2), i32(2), 16, 4, 5), "query_start_loc"),
        (lambda: P.slot_mapping(i32(2, 3), i32(3), i32(1), 16, 4, 5), "seq_lens"),
        (lambda: P.slot_mapping(i32(2, 3), i32(3), i32(2), 16, 4, 5,
                                out=torch.zeros(4, dtype=torch.int64)), "slot_mapping"),
        (lambda: P.slot_mapping_positions(i32(2, 3), i32(5), torch.zeros(5, dtype=torch.int64),
                                          16, 4, out=torch.zeros(4, dtype=torch.int64)), "out"),
        (lambda: P.rope_cache_write(q, torch.zeros(2, 2, 64), torch.zeros(2, 2, 64), kc, kc,
                                    torch.zeros(1, dtype=torch.int64),
                                    torch.zeros(2, dtype=torch.int64), torch.zeros(8, 64)),
         "slot_mapping"),
        (lambda: P.rope_cache_write(q, torch.zeros(2, 2, 64), torch.zeros(2, 2, 64), kc, kc,
                                    torch.zeros(2, dtype=torch.int64),
                                    torch.zeros(1, dtype=torch.int64), torch.zeros(8, 64)),
         "positions"),
    ]
    for call, name in cases:
        with pytest.raises(ValueError, match=rf"^{name} must (be a \d-D tensor with at least|"
                                             rf"have shape)"):
            call()
    # a decode step's new rows: one per request, of the cache's input dtype
    for k in (torch.zeros(3, 2, 64), torch.zeros(2, 1, 64),
              torch.zeros(2, 2, 64, dtype=torch.bfloat16)):
        with pytest.raises(ValueError, match=r"^k must be \[num_seqs, num_kv_heads, head_dim\]"):
            P.decode_step(q, k, kv, kc, kc, i32(2, 3), i32(2), 0.1)


def _header_text():
    return re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)


def test_binding_constants_match_the_header():
    from paged_kv_cache_434_b200 import binding as B
    text = _header_text()
    enums = dict((k, int(v)) for k, v in re.findall(r"\b(PA_[A-Z0-9_]+)\s*=\s*(\d+)", text))
    for name in ("PA_OK", "PA_ERR_INVALID_ARG", "PA_ERR_UNSUPPORTED", "PA_ERR_WORKSPACE",
                 "PA_ERR_CUDA", "PA_ERR_DEVICE_OOB", "PA_ERR_TIMEOUT", "PA_F32", "PA_BF16",
                 "PA_FP8_E4M3"):
        assert getattr(B, name) == enums[name], name
    defines = dict(re.findall(r"#define\s+(PA_[A-Z0-9_]+)\s+\(?([0-9a-fx]+)", text))
    bits = {k: int(v, 0) for k, v in defines.items() if k.startswith("PA_ERRBIT_")}
    assert bits and all(getattr(B, k[3:]) == v for k, v in bits.items()), bits
    assert B.DECODE_NO_ALLOC_MAX_BYTES == 32 << 20
    assert "(32u << 20)" in text.split("PA_DECODE_NO_ALLOC_MAX_BYTES", 1)[1].splitlines()[0]
    assert len(B.TIMED_KERNELS) == int(defines["PA_TIMED_KERNELS"])
    for i, name in enumerate(B.TIMED_KERNELS):
        assert int(defines[f"PA_TK_{name.upper()}"]) == i


_CTYPES_OF = {"int32_t": "c_int", "int64_t": "c_long", "float": "c_float", "double": "c_double",
              "uint32_t": "c_uint",
              "size_t": "c_ulong", "int": "c_int"}


def _kind(ctype):
    """Comparable name of a ctypes argument type."""
    import ctypes
    if ctype is ctypes.c_void_p:
        return "ptr"
    if isinstance(ctype, type) and issubclass(ctype, ctypes._Pointer):
        from paged_kv_cache_434_b200.binding import CacheDesc
        return "desc_ptr" if ctype._type_ is CacheDesc else "ptr"
    if ctype is ctypes.c_char_p:
        return "str"
    return ctype.__name__


def test_binding_signatures_match_the_header():
    """Argument count and kind of every ctypes prototype against the C
    prototype in include/pa.h (pointers, 32/64-bit integers, floats)."""
    import ctypes
    from paged_kv_cache_434_b200 import binding as B
    text = _header_text()
    protos = dict(re.findall(r"\b(?:pa_status|size_t|int|const char\*)\s+(pa_[a-z_]+)\(([^)]*)\)",
                             text, flags=re.S))
    assert set(protos) == set(B.EXPORTS)
    for name, params in protos.items():
        want = []
        for p in filter(None, (x.strip() for x in params.split(","))):
            if p == "void":
                continue
            if "pa_cache_desc" in p and "*" in p:
                want.append("desc_ptr")
            elif "*" in p:
                want.append("ptr")
            else:
                base = p.rsplit(None, 1)[0].replace("const ", "").strip()
                want.append(getattr(ctypes, _CTYPES_OF[base]).__name__)
        got = [_kind(t) for t in B._SIGNATURES[name][0]]
        assert got == want, (name, got, want)


def test_cache_desc_layout_matches_the_c_struct(tmp_path):
    """Size and field offsets of pa_cache_desc as gcc lays it out, against the
    ctypes structure the binding passes by pointer."""
    import ctypes
    import shutil
    import subprocess
    from paged_kv_cache_434_b200.binding import CacheDesc
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    names = [n for n, _ in CacheDesc._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"pa.h\"\nint main(void) {\n"
                   "  printf(\"%zu\\n\", sizeof(pa_cache_desc));\n" +
                   "".join(f"  printf(\"%zu\\n\", offsetof(pa_cache_desc, {n}));\n" for n in names) +
                   "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    assert got[0] == ctypes.sizeof(CacheDesc)
    assert got[1:] == [getattr(CacheDesc, n).offset for n in names]


def test_plain_c_program_links_and_calls_the_library(tmp_path, lib):
    """The boundary is usable from C alone: a C99 program including only
    include/pa.h links libpa_b200.so and gets the documented statuses from
    calls that are refused on the host (nothing reaches a device)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    libdir = os.path.join(ROOT, "paged_kv_cache_434_b200", "lib")
    src = tmp_path / "client.c"
    src.write_text(r'''
#include <stdio.h>
#include "pa.h"
int main(void) {
  pa_cache_desc d = {16, 16, 2, 64, PA_BF16, 1.0f, 1.0f};
  pa_cache_desc bad = d;
  bad.head_dim = 96;
  printf("%d\n", pa_version() >= 100);
  printf("%s\n", pa_status_str(PA_ERR_WORKSPACE));
  printf("%d\n", pa_decode_workspace_size(4, 8, 3, &d) > 0);
  printf("%d\n", (int)pa_cache_write(NULL, NULL, NULL, NULL, NULL, 4, &d, NULL, NULL));
  printf("%d\n", (int)pa_cache_write(NULL, NULL, NULL, NULL, NULL, 1, &bad, NULL, NULL));
  printf("%d\n", (int)pa_decode(NULL, NULL, NULL, NULL, NULL, 0.1f, NULL, 0, 8, 3, PA_F32, &d,
                                NULL, 0, NULL, NULL));
  return 0;
}
''')
    exe = tmp_path / "client"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-L", libdir,
                    "-lpa_b200", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    assert out[0] == "1"
    assert out[1] == "workspace missing, misaligned or too small"
    assert out[2] == "1"
    assert out[3:6] == ["1", "2", "0"]   # INVALID_ARG, UNSUPPORTED, OK (nothing to do)

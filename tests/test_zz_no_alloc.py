"""pa_decode_no_alloc against the fp64 oracle and against pa_decode, through
the C ABI.

pa_decode_no_alloc serves callers that can't allocate device memory (a
plug-in inside an engine that owns every allocation, a runtime that forbids
cudaMalloc after start-up): it runs the same decode kernels on a static
device scratch array inside the library instead of a caller workspace.  Its
`late` mark runs this file after every other test, so that a run stopping at
its first failure has already run them; it also passes alone in a fresh
process.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import binding as B
from paged_kv_cache_434_b200 import workloads as W

from _util import assert_close, f64, oracle_full

pytestmark = [pytest.mark.gpu, pytest.mark.late(9)]


@pytest.mark.parametrize("dtype,hq,hkv,d,lens", [
    ("bf16", 32, 8, 128, [4000, 1, 17, 2500, 813, 64, 3333, 129]),
    ("bf16", 8, 1, 128, [900, 1, 33, 2100, 16]),
    ("f32", 8, 2, 64, [25, 9, 40, 700, 1]),
])
def test_no_alloc_matches_oracle_and_pa_decode_on_two_calls_in_a_row(cuda_device, dtype, hq,
                                                                     hkv, d, lens):
    w = W.custom("no_alloc", lens, [1] * len(lens), hq, hkv, d, 16, dtype, seed=21)
    host = W.make_tensors(w, "cpu", where="host")
    t = {k: v.to(cuda_device) for k, v in host.items()}
    idx = W.index_tensors(w, cuda_device)
    assert P.decode_workspace_size(w.num_seqs, hq, w.max_blocks_per_seq, t["k_cache"]) \
        <= B.DECODE_NO_ALLOC_MAX_BYTES
    # the step's own cache write first (through the library), then attention
    # over the written pools; the oracle does the same on the host copies
    slots = P.slot_mapping(idx["block_tables"], idx["query_start_loc"], idx["seq_lens"],
                           w.block_size, w.num_blocks, w.num_tokens)
    P.cache_write(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], slots)
    _, _, _, oracle_out, _, valid = oracle_full(w, host)
    ref = P.decode(t["q"], t["k_cache"], t["v_cache"], idx["block_tables"], idx["seq_lens"],
                   w.scale)
    err = P.new_error_word(cuda_device)
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        B.decode_no_alloc(t["q"], t["k_cache"], t["v_cache"], idx["block_tables"],
                          idx["seq_lens"], w.scale, out, err=err)
        torch.cuda.synchronize()
        assert P.read_error(err) == 0
        assert_close(f64(out), f64(ref), dtype, f"no-alloc call {call} vs pa_decode")
        assert_close(f64(out)[valid], oracle_out[valid], dtype, f"no-alloc call {call} vs oracle")


def test_no_alloc_rejects_problems_beyond_its_scratch(cuda_device):
    # 4096 requests of up to 64K tokens need far more than the static scratch
    kc = torch.empty(1, 16, 8, 128, dtype=torch.bfloat16, device=cuda_device)
    need = P.decode_workspace_size(4096, 32, 4096, kc)
    assert need > B.DECODE_NO_ALLOC_MAX_BYTES
    q = torch.zeros(4096, 32, 128, dtype=torch.bfloat16, device=cuda_device)
    tables = torch.zeros(4096, 4096, dtype=torch.int32, device=cuda_device)
    lens = torch.ones(4096, dtype=torch.int32, device=cuda_device)
    out = torch.empty(4096, 32, 128, device=cuda_device)
    with pytest.raises(B.PagedAttentionError) as e:
        B.decode_no_alloc(q, kc, kc, tables, lens, 0.1, out)
    assert e.value.status == B.PA_ERR_WORKSPACE

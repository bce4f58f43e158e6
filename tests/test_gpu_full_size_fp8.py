"""Full-size parity of the decode workloads over e4m3 pools (scale 1/56):
the Llama-3-8B batch (64 requests of 512-8192 tokens) and the long-context
split-KV batch (32K, 64K, 96K and 128K tokens), drawn and launched as the
benchmark draws and launches them.

Checked against the oracle, through the same step the benchmark times:
  * the slot of every new token, bit for bit;
  * the codes of every written row, bit for bit against the oracle's
    quantisation of the new K/V rows;
  * a sample of unwritten rows, unchanged;
  * attention on every row of every request, against the fp64 oracle over
    the pools' dequantised values, within the bf16-input tolerance.

The `late` mark runs this file after the parity suites.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import workloads as W
from _util import assert_close, device_blocks, f64, oracle_request

pytestmark = [pytest.mark.gpu, pytest.mark.late(1)]


def _full_size_fp8(w, dev, reqs):
    assert w.kv_dtype == "fp8"
    t = W.make_tensors(w, dev, where="device")
    idx = W.index_tensors(w, dev)
    Hkv, D = w.num_kv_heads, w.head_dim
    kc = t["k_cache"].view(torch.uint8)
    vc = t["v_cache"].view(torch.uint8)
    blocks = device_blocks(w, (t["k_cache"], t["v_cache"]), reqs)
    # untouched-row sample, taken before the step
    gen = np.random.default_rng(99)
    probe = torch.from_numpy(gen.integers(0, w.num_blocks * w.block_size, 4096)).to(dev)
    kc_rows = kc.view(-1, Hkv, D)
    vc_rows = vc.view(-1, Hkv, D)
    before = kc_rows.index_select(0, probe).clone()

    err = P.new_error_word(dev)
    slots = torch.empty(w.num_tokens, dtype=torch.int64, device=dev)
    out = P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
                 idx["query_start_loc"], idx["seq_lens"], w.scale, decode_only=w.is_decode,
                 out_dtype=torch.float32, slots=slots, err=err, kv_scales=w.kv_scales)
    torch.cuda.synchronize()
    assert P.read_error(err) == 0

    ref_slots = oracle.slot_mapping(w.block_tables, w.query_start_loc, w.seq_lens, w.block_size)
    assert np.array_equal(slots.cpu().numpy(), ref_slots)
    k_codes = oracle.quantize(f64(t["k_new"]).astype(np.float32), w.kv_scale)
    v_codes = oracle.quantize(f64(t["v_new"]).astype(np.float32), w.kv_scale)
    assert np.array_equal(kc_rows.index_select(0, slots).cpu().numpy(), k_codes)
    assert np.array_equal(vc_rows.index_select(0, slots).cpu().numpy(), v_codes)
    written = set(ref_slots.tolist())
    keep = torch.tensor([i for i, s in enumerate(probe.tolist()) if s not in written], device=dev)
    assert torch.equal(kc_rows.index_select(0, probe)[keep], before[keep])

    # every row of the chosen requests; the oracle quantises the new rows and
    # attends over the values the codes stand for
    k_new, v_new, q = t["k_new"].cpu(), t["v_new"].cpu(), t["q"].cpu()
    qsl = w.query_start_loc
    got, ref = [], []
    for b in reqs:
        ref.append(oracle_request(w, blocks.pop(int(b)), k_new, v_new, q, int(b),
                                  dequant=lambda c: oracle.dequantize(c, w.kv_scale)))
        got.append(f64(out[int(qsl[b]):int(qsl[b + 1])]))
    return assert_close(np.concatenate(got), np.concatenate(ref), "bf16", w.name)


def test_full_llama8b_decode_fp8(cuda_device):
    w = W.llama8b_decode_fp8(0)
    _full_size_fp8(w, cuda_device, range(w.num_seqs))     # all 64 requests


def test_full_long_context_fp8(cuda_device):
    _full_size_fp8(W.long_context_decode_fp8(0), cuda_device, [0, 1, 2, 3])

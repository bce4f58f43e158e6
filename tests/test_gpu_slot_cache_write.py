"""pa_slot_mapping_cache_write: slot mapping and the cache write in one launch.
It must give what the two separate calls give -- the same slots, the same
pools bit for bit and the same error bits -- and so match the oracle's slot
function and cache write ("AI Infra入门干货总结：大模型是如何高效推理的",
sections "Paged Attention" and "Reshape & Cache")."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import workloads as W
from _util import bits, f64, fp8_codes

pytestmark = pytest.mark.gpu


def _two_calls(w, t, idx, err):
    slots = P.slot_mapping(idx["block_tables"], idx["query_start_loc"], idx["seq_lens"],
                           w.block_size, w.num_blocks, w.num_tokens, err=err)
    P.cache_write(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], slots, err=err,
                  kv_scales=w.kv_scales)
    return slots


def _fused(w, t, idx, err, decode_form):
    qsl = None if decode_form else idx["query_start_loc"]
    return P.slot_mapping_cache_write(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
                                      idx["block_tables"], qsl, idx["seq_lens"], err=err,
                                      kv_scales=w.kv_scales)


def _pool(x):
    return fp8_codes(x) if x.dtype == torch.float8_e4m3fn else bits(x)


def _compare(w, dev, decode_form=False):
    host = W.make_tensors(w, "cpu", where="host")
    idx = W.index_tensors(w, dev)
    a = {k: v.to(dev) for k, v in host.items()}
    b = {k: v.to(dev) for k, v in host.items()}
    ea, eb = P.new_error_word(dev), P.new_error_word(dev)
    sa = _two_calls(w, a, idx, ea)
    sb = _fused(w, b, idx, eb, decode_form)
    torch.cuda.synchronize()
    assert P.read_error(eb) == P.read_error(ea)
    assert torch.equal(sa, sb)
    for name in ("k_cache", "v_cache"):
        assert np.array_equal(_pool(a[name]), _pool(b[name])), name
    # and the oracle's slot function on the same requests
    ref = oracle.slot_mapping(w.block_tables, w.query_start_loc, w.seq_lens, w.block_size)
    assert np.array_equal(sb.cpu().numpy(), ref)
    return host, b


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_decode_step_without_offsets(cuda_device, dtype, bs):
    lens = [1, bs, bs + 1, 300, 1000, 77]
    w = W.custom(f"scw_dec_{dtype}_{bs}", lens, [1] * len(lens), 8, 2, 64, bs, dtype, seed=bs)
    host, b = _compare(w, cuda_device, decode_form=True)
    ref_slots = oracle.slot_mapping(w.block_tables, w.query_start_loc, w.seq_lens, w.block_size)
    kc, vc, _ = oracle.cache_write(f64(host["k_cache"]), f64(host["v_cache"]),
                                   f64(host["k_new"]), f64(host["v_new"]), ref_slots)
    assert np.array_equal(f64(b["k_cache"]), kc) and np.array_equal(f64(b["v_cache"]), vc)


@pytest.mark.parametrize("n_decodes,geom", [(3, (32, 8, 128)), (40, (32, 8, 128)),
                                             (700, (8, 2, 64))])
def test_mixed_step_offsets(cuda_device, n_decodes, geom):
    """Chunks and decodes in one flattened step; with 700 requests the token ->
    request search takes more than one round of 32 probes."""
    hq, hkv, d = geom
    rng = np.random.default_rng(n_decodes)
    lens = [300, 17, 1024] + [int(x) for x in rng.integers(1, 900, n_decodes)]
    qlens = [64, 9, 200] + [1] * n_decodes
    w = W.custom(f"scw_mixed_{n_decodes}", lens, qlens, hq, hkv, d, 16, "bf16", seed=n_decodes)
    _compare(w, cuda_device)


def test_empty_requests_are_passed_over(cuda_device):
    """Requests with no new token (equal offsets) own no token of the step."""
    dev = cuda_device
    w = W.custom("scw_empty", [40, 30, 55, 20], [2, 1, 3, 1], 8, 2, 64, 16, "f32", seed=4)
    host = W.make_tensors(w, "cpu", where="host")
    idx = W.index_tensors(w, dev)
    t = {k: v.to(dev) for k, v in host.items()}
    # make request 1 empty: offsets [0, 2, 2, 5, 6] -> its token goes to request 2
    qsl = torch.tensor([0, 2, 2, 5, 6], dtype=torch.int32, device=dev)
    seq_lens = idx["seq_lens"].clone()
    err = P.new_error_word(dev)
    slots = P.slot_mapping_cache_write(t["k_new"][:6], t["v_new"][:6], t["k_cache"], t["v_cache"],
                                       idx["block_tables"], qsl, seq_lens, err=err)
    ref = P.slot_mapping(idx["block_tables"], qsl, seq_lens, w.block_size, w.num_blocks, 6,
                         err=P.new_error_word(dev))
    torch.cuda.synchronize()
    assert P.read_error(err) == 0
    assert torch.equal(slots, ref)


def test_fp8_pools(cuda_device):
    lens = [40, 300, 77, 1]
    w = W.with_fp8_cache(W.custom("scw_fp8", lens, [1] * len(lens), 8, 2, 128, 16, "bf16",
                                  seed=91))
    _compare(w, cuda_device, decode_form=True)
    _compare(w, cuda_device, decode_form=False)


def test_error_bits_match_the_two_calls(cuda_device):
    """A block id outside the pool, a seq_len longer than the table and a query
    longer than its sequence: the same slots (-1) and error bits as
    pa_slot_mapping + pa_cache_write, and nothing written for those tokens."""
    dev = cuda_device
    w = W.custom("scw_err", [20, 20, 20, 20], [1, 1, 1, 1], 8, 2, 64, 16, "f32", seed=15,
                 extra_blocks=1)
    host = W.make_tensors(w, "cpu", where="host")
    idx = W.index_tensors(w, dev)
    tables = idx["block_tables"].clone()
    tables[1, 1] = w.num_blocks + 5            # request 1's token (position 19) is in column 1
    lens_a = idx["seq_lens"].clone()
    lens_a[2] = 20 + 16 * 5                    # request 2: longer than its table
    qsl_a = torch.tensor([0, 1, 2, 3, 4], dtype=torch.int32, device=dev)
    lens_b = idx["seq_lens"].clone()
    lens_b[1] = 1                              # request 1: two new tokens, seq_len 1
    qsl_b = torch.tensor([0, 1, 3, 3, 4], dtype=torch.int32, device=dev)  # request 2: none
    for qsl, lens, want in ((qsl_a, lens_a, P.ERRBIT_BLOCK_OOB | P.ERRBIT_SEQ_TOO_LONG),
                            (qsl_b, lens_b, P.ERRBIT_QUERY_TOO_LONG)):
        a = {k: v.to(dev) for k, v in host.items()}
        b = {k: v.to(dev) for k, v in host.items()}
        ea, eb = P.new_error_word(dev), P.new_error_word(dev)
        sa = P.slot_mapping(tables, qsl, lens, w.block_size, w.num_blocks, 4, err=ea)
        P.cache_write(a["k_new"][:4], a["v_new"][:4], a["k_cache"], a["v_cache"], sa, err=ea)
        sb = P.slot_mapping_cache_write(b["k_new"][:4], b["v_new"][:4], b["k_cache"],
                                        b["v_cache"], tables, qsl, lens, err=eb)
        torch.cuda.synchronize()
        bits_a, bits_b = P.read_error(ea), P.read_error(eb)
        assert bits_a == want and bits_b == want
        assert torch.equal(sa, sb) and int((sb < 0).sum()) > 0
        assert torch.equal(a["k_cache"], b["k_cache"]) and torch.equal(a["v_cache"], b["v_cache"])


def test_decode_form_needs_one_token_per_request(cuda_device):
    dev = cuda_device
    w = W.custom("scw_shape", [20, 30], [1, 1], 8, 2, 64, 16, "f32", seed=2)
    host = W.make_tensors(w, "cpu", where="host")
    idx = W.index_tensors(w, dev)
    t = {k: v.to(dev) for k, v in host.items()}
    k3 = torch.cat([t["k_new"], t["k_new"][:1]])
    v3 = torch.cat([t["v_new"], t["v_new"][:1]])
    with pytest.raises(ValueError):
        P.slot_mapping_cache_write(k3, v3, t["k_cache"], t["v_cache"], idx["block_tables"], None,
                                   idx["seq_lens"])

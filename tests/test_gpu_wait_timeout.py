"""A bounded device wait that runs out ends by itself, reports
PA_ERRBIT_TIMEOUT through the error word, and leaves the context usable.

Every mbarrier wait in the attention kernels is bounded by time; in a correct
call none runs out.  pa_selftest_wait_timeout drives the same bounded-wait
routine against an mbarrier that nothing arrives at, with a limit of a few
milliseconds.  The test then runs a normal decode call and checks it against
the fp64 oracle, which shows that the timeout left the device working.
"""

import pytest
import torch

import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import binding as B
from paged_kv_cache_434_b200 import workloads as W

from _util import assert_close, f64, oracle_full

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_us", [2000, 20000])
def test_wait_runs_out_and_sets_the_timeout_bit(cuda_device, limit_us):
    err = P.new_error_word(cuda_device)
    waited = torch.zeros(1, dtype=torch.int64, device=cuda_device)
    B.selftest_wait_timeout(limit_us, err, waited)
    torch.cuda.synchronize()
    assert P.read_error(err) == B.ERRBIT_TIMEOUT
    ns = int(waited.item())
    # the wait gives up only once its limit has passed, and soon after it
    assert limit_us * 1000 <= ns < limit_us * 1000 + 50_000_000
    # the error word was cleared by the read: a second read finds nothing
    assert P.read_error(err) == 0

    # the context still runs a normal call, and its result is exact
    w = W.tiny_decode(seed=3)
    host = W.make_tensors(w, "cpu", where="host")
    t = {k: v.to(cuda_device) for k, v in host.items()}
    idx = W.index_tensors(w, cuda_device)
    out = P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
                 idx["query_start_loc"], idx["seq_lens"], w.scale, decode_only=True, err=err)
    torch.cuda.synchronize()
    assert P.read_error(err) == 0
    _, _, _, ref, _, valid = oracle_full(w, host)
    assert_close(f64(out)[valid], ref[valid], "f32", "decode after a timeout")


def test_limit_outside_its_range_is_refused(cuda_device):
    err = P.new_error_word(cuda_device)
    for bad in (0, 100001):
        with pytest.raises(B.PagedAttentionError) as e:
            B.selftest_wait_timeout(bad, err)
        assert e.value.status == B.PA_ERR_INVALID_ARG


def test_read_error_status_names_the_condition(cuda_device):
    """pa_read_error's status: PA_ERR_TIMEOUT once a wait gave up (whatever
    other bits are set), PA_ERR_DEVICE_OOB for out-of-range input alone, PA_OK
    for a clean word; the bits come back either way."""
    import ctypes

    def status(word):
        bits = ctypes.c_int32(0)
        st = B._lib().pa_read_error(ctypes.c_void_p(word.data_ptr()), ctypes.byref(bits),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        return st, bits.value

    err = P.new_error_word(cuda_device)
    B.selftest_wait_timeout(1000, err)
    err.add_(B.ERRBIT_BLOCK_OOB)          # queued after the wait on the same stream
    assert status(err) == (B.PA_ERR_TIMEOUT, B.ERRBIT_TIMEOUT | B.ERRBIT_BLOCK_OOB)
    err.fill_(B.ERRBIT_SEQ_TOO_LONG)
    assert status(err) == (B.PA_ERR_DEVICE_OOB, B.ERRBIT_SEQ_TOO_LONG)
    assert status(err) == (B.PA_OK, 0)

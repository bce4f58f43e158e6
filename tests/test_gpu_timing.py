"""Per-launch event timing of an attention call (a measurement aid): timed
calls give the same output as untimed ones, and report a positive device
time for each launch they made."""

import numpy as np
import pytest
import torch

import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", ["decode", "mixed"])
def test_timed_call_matches_untimed(cuda_device, kind):
    dev = cuda_device
    qlens = [1, 1, 1, 1] if kind == "decode" else [1, 9, 200, 1]
    w = W.custom(f"timing_{kind}", [300, 17, 1024, 5], qlens, 32, 8, 128, 16, "bf16", seed=3)
    host = W.make_tensors(w, "cpu", where="host")
    t = {k: v.to(dev) for k, v in host.items()}
    idx = W.index_tensors(w, dev)

    def call():
        err = P.new_error_word(dev)
        out = P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
                     idx["block_tables"], idx["query_start_loc"], idx["seq_lens"], w.scale,
                     decode_only=w.is_decode, err=err)
        torch.cuda.synchronize()
        assert P.read_error(err) == 0
        return out.cpu()

    plain = call()
    P.kernel_timing(True)
    try:
        timed = call()
        ms = P.kernel_times()
        with pytest.raises(P.PagedAttentionError):
            P.kernel_times()          # read once per timed call
    finally:
        P.kernel_timing(False)
    with pytest.raises(P.PagedAttentionError):
        P.kernel_times()              # timing off
    assert np.array_equal(plain.view(torch.int32).numpy(), timed.view(torch.int32).numpy())
    for k in ("plan", "decode", "merge"):
        assert k in ms and 0.0 < ms[k] < 1e3
    if kind == "mixed":
        assert "tiles" in ms and ms["tiles"] > 0.0

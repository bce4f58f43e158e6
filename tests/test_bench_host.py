"""The benchmark's host side (no GPU): the algorithmic counts -- prefill
FLOPs, unique K/V bytes with shared blocks counted once, the decode-launch
bytes, the fused RoPE + cache write bytes, checked against direct sums over
the workloads' definitions."""

import numpy as np

import bench
from paged_kv_cache_434_b200 import workloads as W


def test_prefill_flops_of_the_mixed_step():
    w = W.mixed_step(0)
    # two chunks: 2048 queries after 4096 cached keys, and a fresh 2048-token prompt;
    # query i of a chunk sees prefix + i + 1 keys; 4 * D * Hq FLOPs per visible pair
    per_pair = 4 * 128 * 32
    a = sum(4096 + i + 1 for i in range(2048)) * per_pair
    b = sum(i + 1 for i in range(2048)) * per_pair
    assert bench.prefill_flops(w) == a + b
    assert abs((a + b) - 2.06e11) / 2.06e11 < 0.01


def test_unique_kv_bytes_count_shared_blocks_once():
    w = W.shared_prefix_decode(0)
    row = 2 * w.num_kv_heads * w.head_dim * w.elt_bytes
    prefix = w.shared_prefix_blocks * w.block_size
    suffix = int((w.seq_lens.astype(np.int64) - prefix).sum())
    assert W.kv_bytes_touched(w, unique=True) == (prefix + suffix) * row
    assert W.kv_bytes_touched(w, unique=False) == int(w.seq_lens.astype(np.int64).sum()) * row
    # the decode launch streams only the suffixes (the prefix goes to the tiles)
    qo = w.num_seqs * w.num_heads * w.head_dim * (w.elt_bytes + 4)
    assert bench.decode_kernel_bytes(w) == suffix * row + qo


def test_decode_bytes_of_a_plain_batch():
    w = W.llama8b_decode(0)
    row = 2 * 8 * 128 * 2
    kv = int(w.seq_lens.astype(np.int64).sum()) * row
    bc = bench.byte_counts(w)
    assert bc["kv"] == kv
    assert bc["attention"] == kv + 64 * 32 * 128 * 2 + 64 * 32 * 128 * 4
    assert bench.decode_kernel_bytes(w) == bc["attention"]
    # the FP8 cache halves the K/V bytes of the same batch
    f = W.llama8b_decode_fp8(0)
    assert W.kv_bytes_touched(f) * 2 == kv


def test_rope_write_bytes():
    w = W.mixed_step(0)
    T = w.num_tokens
    per_token = 2 * 32 * 128 * 2 + 4 * 8 * 128 * 2 + 128 * 4 + 16
    assert bench.rope_bytes(w) == T * per_token


def test_job_throughput_is_weak_scaling_over_the_slowest_rank():
    assert bench.job_throughput(1e9, 10, 8, 2.0) == 1e9 * 10 * 8 / 2.0


def test_own_peaks_never_costs_the_benchmark_line(monkeypatch):
    """The bench's own copy / GEMM reference rates are context: where they
    cannot be measured the result says why instead of raising.  (CUDA events
    are made to fail, so the test means the same with or without a GPU.)"""
    import torch

    def no_events(*a, **k):
        raise RuntimeError("no CUDA events here")

    monkeypatch.setattr(torch.cuda, "Event", no_events)
    r = bench.own_peaks(torch.device("cpu"), copy_bytes=1 << 20, gemm_n=64, iters=1)
    assert set(r) == {"error"} and r["error"]


def test_default_line_carries_every_decode_config(monkeypatch, capsys):
    """The default run's one JSON line: the Llama-3-8B decode headline plus the
    mixed step (the metric's second half), the shared-prefix and the
    long-context batches, each measured in the same process (measure() is
    stubbed here: only the line's assembly is checked)."""
    import json
    import types

    def fake_measure(args, name, rank, world, local, with_e2e=True, with_cpu=True):
        roof = {"bound": "hbm", "frac": 1.0, "attention_call": {"ms": 1.0, "frac": 0.9}}
        return {"metric": name, "value": 1.0, "unit": "u", "ms_per_step": 1.0, "e2e": {},
                "kernel_ms": {"tiles": 0.5}, "gpu_launches": 4, "clocks": {},
                "roofline": roof, "without_cache_write": {"value": 1.0},
                "prefill_roofline": {"frac": 0.5},
                "config": {"workload": name, "num_seqs": 1, "num_tokens": 1,
                           "prefill_flops_per_step": 1e9, "num_heads": 1, "num_kv_heads": 1,
                           "block_size": 16, "kv_bytes_unique": 1}}

    monkeypatch.setattr(bench, "measure", fake_measure)
    monkeypatch.setattr(bench.torch.cuda, "empty_cache", lambda: None)
    args = types.SimpleNamespace(workload="llama8b_decode", no_extras=False)
    bench.run_ours(args, 0, 1, 0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["metric"] == "llama8b_decode"
    for key, name in (("mixed_step", "mixed"), ("shared_prefix", "shared_prefix"),
                      ("long_context", "long_context")):
        assert line[key]["metric"] == name and line[key]["config"]["workload"] == name
    assert line["mixed_step"]["prefill_roofline"]["alone"] == {"frac": 0.5}
    assert line["shared_prefix"]["attention_call"]["frac"] == 0.9
    assert line["long_context"]["roofline"]["attention_call"]["frac"] == 0.9

"""Benchmark: one layer's paged-KV attention step on synthetic, seeded inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is the whole hot path for one batch: slot mapping of the new tokens,
the cache write (reshape_and_cache) and the attention call (pa_decode for
decode batches, pa_mixed_step for a chunked-prefill step).  Inputs are
resident in HBM when timing starts; L2 is flushed (a 512 MiB write, then a
512 MiB read, so no dirty line is written back during the step) before
every step and only the step itself sits between its CUDA events.  With
torchrun (N > 1) every rank runs its own batch on its own GPU (sequences are
independent: weak scaling, no collective on the data path); the time is the
max over ranks.  Rank 0 prints one JSON line.

--workload rope_write times the step just upstream instead: slot mapping and
the rotary embedding of Q/K fused with the cache write, for the 8192 new
tokens of the mixed chunked-prefill step (Llama-3-8B geometry, rope_theta
500000).

--workload cow_copy times copy-on-write block copies: 2048 (source,
destination) pairs of 16-token blocks in Llama-3-8B layer pools (8 KV heads,
head_dim 128, bf16; 8192 blocks per pool).

--workload graph_decode times a small decode step (4 requests, Llama-3-8B
geometry) captured once in a CUDA graph and replayed, beside the same step
launched eagerly: launch overhead is what a graph removes.

--impl reference times the CPU oracle (float64 NumPy, the test reference) on
a bounded sample of the same workload, on this host's cores.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    "tiny": ("tiny_decode", 1),
    "llama8b_decode": ("llama8b_decode", 2),
    "long_context": ("long_context_decode", 3),
    "mixed": ("mixed_step", 4),
    "shared_prefix": ("shared_prefix_decode", 5),
    "mixed_prefill": ("mixed_step_prefill_only", 4),
    "llama8b_decode_fp8": ("llama8b_decode_fp8", 2),   # the same batch over e4m3 pools
    "long_context_fp8": ("long_context_decode_fp8", 3),
    "rope_write": ("mixed_step", 4),   # the mixed step's 8192 new tokens, fused RoPE + cache write
    "cow_copy": ("llama8b_decode", 2),  # copy-on-write block copies in Llama-3-8B layer pools
    "graph_decode": ("llama8b_decode", 2),  # a small decode step replayed from a CUDA graph
}
FLUSH_BYTES = 512 << 20
L2_NOTE = ("flushed before every step, outside the events: a 512 MiB write, then a 512 MiB "
           "read, so that L2 holds clean lines and no write-back of the flush competes with "
           "the step")


class L2Flush:
    """Evicts L2 between steps: writes a buffer larger than L2, then reads
    another, so that the dirty lines of the write are written back before the
    step instead of during it."""

    def __init__(self, dev):
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(FLUSH_BYTES // 8, dtype=torch.int64, device=dev)

    def fill_(self, v=1):
        self.w.fill_(v)
        self.r.sum()


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="llama8b_decode", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="time budget of the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="default workload only: skip the mixed-step and shared-prefix objects")
    return ap.parse_args(argv)


def dist_setup():
    """Rank, world size and local rank from the torchrun environment; with more
    than one rank, a process group (NCCL on GPUs; gloo where no GPU is present,
    which only the host-side tests use) with a short timeout."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout,
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    return rank, world, local


def job_throughput(units_per_step: float, steps: int, world: int, max_total_s: float) -> float:
    """Whole-job rate: every rank processed `units_per_step` each step (weak
    scaling), divided by the slowest rank's timed seconds."""
    return units_per_step * steps * world / max_total_s


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, dev) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def own_peaks(dev, copy_bytes: int = 1 << 30, gemm_n: int = 8192, iters: int = 10):
    """This process's own reference rates, reported as context beside the
    measured peaks: a device-to-device copy (read + write bytes over time) and
    a bf16 torch matmul (2 n^3 FLOP), each timed with CUDA events after three
    warm-up runs.  Never raises: a failure is reported in the result."""
    try:
        stream = torch.cuda.current_stream()
        a = torch.empty(copy_bytes, dtype=torch.uint8, device=dev)
        b = torch.empty_like(a)

        def timed(fn):
            for _ in range(3):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(iters):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / 1e3 / iters

        copy_s = timed(lambda: b.copy_(a))
        del a, b
        x = torch.randn(gemm_n, gemm_n, device=dev).to(torch.bfloat16)
        y = torch.randn(gemm_n, gemm_n, device=dev).to(torch.bfloat16)
        z = torch.empty(gemm_n, gemm_n, dtype=torch.bfloat16, device=dev)
        gemm_s = timed(lambda: torch.matmul(x, y, out=z))
        del x, y, z
        return {"copy_gbs": round(2 * copy_bytes / copy_s / 1e9, 1),
                "bf16_gemm_tflops": round(2 * gemm_n ** 3 / gemm_s / 1e12, 1),
                "how": f"{copy_bytes >> 20} MiB device-to-device copy, {gemm_n}^3 bf16 "
                       f"torch.matmul; CUDA events, mean of {iters} after 3 warm-up"}
    except Exception as e:  # context only: never costs the benchmark line
        return {"error": f"{type(e).__name__}: {e}"[:200]}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def kernel_traffic(kernel_src: str, profile_md: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current kernel source (the summary records the source's sha256)."""
    path = os.path.join(ROOT, "profiles", profile_md)
    src = os.path.join(ROOT, "paged_kv_cache_434_b200", "csrc", kernel_src)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    vals = {}
    for line in open(path, encoding="utf-8"):
        if ":" in line and line.strip().lstrip("- ").startswith(("kernel_source_sha256",
                                                                  "traffic_bytes_per_launch")):
            k, v = line.split(":", 1)
            m = re.search(r"`([^`]+)`", v)  # the value is the first `quoted` token
            vals[k.strip().lstrip("- ").strip()] = m.group(1) if m else v.strip()
    if vals.get("kernel_source_sha256") != sha:
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev):
        self.proc = None
        self.path = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
        except Exception:
            uuid = None
        self.target = uuid

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.target:
            cmd += ["-i", self.target]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------- workload accounting

def workload_for(name: str, seed: int):
    from paged_kv_cache_434_b200 import workloads as W
    return getattr(W, WORKLOADS[name][0])(seed)


def byte_counts(w, out_elt=4):
    """Algorithmic bytes of one step: unique valid K/V rows once, Q read, O
    written; the cache write reads and writes each new K/V row."""
    from paged_kv_cache_434_b200 import workloads as W
    kv = W.kv_bytes_touched(w, unique=True)
    q = w.num_tokens * w.num_heads * w.head_dim * w.elt_bytes
    o = w.num_tokens * w.num_heads * w.head_dim * out_elt
    cw = 2 * w.num_tokens * w.num_kv_heads * w.head_dim * (w.elt_bytes + w.pool_elt_bytes)
    return {"kv": kv, "q": q, "o": o, "cache_write": cw, "attention": kv + q + o,
            "step": kv + q + o + cw}


def decode_kernel_bytes(w, out_elt=4):
    """Algorithmic bytes of the decode-partition launch: the K/V rows of the
    q_b = 1 requests (valid tokens; a block prefix common to every table is
    left to the tensor-core prefix tiles when the batch has one), their Q rows
    read and their output rows written."""
    row = 2 * w.num_kv_heads * w.head_dim * w.pool_elt_bytes
    dec = [b for b in range(w.num_seqs) if int(w.query_lens[b]) == 1]
    shared = w.shared_prefix_blocks * w.block_size
    toks = sum(int(w.seq_lens[b]) - min(shared, int(w.seq_lens[b])) for b in dec)
    qo = len(dec) * w.num_heads * w.head_dim * (w.elt_bytes + out_elt)
    return toks * row + qo


def prefill_flops(w):
    """Causal-only FLOPs (QK^T and PV, 2 each per MAC) of the q_b > 1 requests."""
    tot = 0
    for b in range(w.num_seqs):
        qb, L = int(w.query_lens[b]), int(w.seq_lens[b])
        if qb > 1:
            keys = sum(L - qb + i + 1 for i in range(qb))
            tot += 4 * w.head_dim * w.num_heads * keys
    return tot


def metric_of(name):
    if name in ("mixed", "mixed_prefill"):
        return "mixed-step query tokens/s per layer", "tokens/s"
    return "paged decode KV GB/s", "GB/s"


# ---------------------------------------------------------------- CPU oracle sample

def oracle_sample(w, pools, seconds: float, rng_seed: int = 0):
    """Time the oracle on whole rows of the workload until `seconds` pass.

    Returns (units_done, elapsed_s, description) where units are KV bytes
    (decode workloads) or query rows (mixed step).
    """
    import oracle
    from threadpoolctl import threadpool_limits
    k_cache, v_cache = pools
    rng = np.random.default_rng(rng_seed)
    qsl = w.query_start_loc
    rows = []
    if w.is_decode:
        order = rng.permutation(w.num_seqs)
        rows = [(int(b), 0) for b in order]
    else:
        dec = [b for b in range(w.num_seqs) if w.query_lens[b] == 1]
        pre = [(b, i) for b in range(w.num_seqs) if w.query_lens[b] > 1
               for i in range(int(w.query_lens[b]))]
        rng.shuffle(dec)
        pi = rng.permutation(len(pre))
        # same mix of prefill and decode rows as the step
        for a, b in zip(pi, dec):
            rows.append(pre[a])
            rows.append((b, 0))
    row_kv = 2 * w.num_kv_heads * w.head_dim * w.pool_elt_bytes
    # fetch the blocks for up to a generous number of rows first (not timed)
    prepared = []
    cache = {}
    for (b, i) in rows[:4096]:
        if b not in cache:
            n = (int(w.seq_lens[b]) + w.block_size - 1) // w.block_size
            ids = torch.from_numpy(w.block_tables[b, :n].astype(np.int64)).to(k_cache.device)
            cache[b] = (k_cache.index_select(0, ids).cpu(), v_cache.index_select(0, ids).cpu())
            if len(cache) > 256:
                break
        prepared.append((b, i))
    q = torch.randn(1, w.num_heads, w.head_dim).to(torch.bfloat16 if w.dtype == "bf16"
                                                     else torch.float32)
    threads = os.cpu_count() or 1
    done_units, t0 = 0, time.perf_counter()
    with threadpool_limits(limits=threads):
        for (b, i) in prepared:
            if b not in cache:
                break
            kb, vb = cache[b]
            L, qb = int(w.seq_lens[b]), int(w.query_lens[b])
            pos = L - qb + i
            table = np.arange(kb.shape[0])
            if w.kv_dtype == "fp8":
                kd = oracle.dequantize(kb.view(torch.uint8).numpy(), w.kv_scale)
                vd = oracle.dequantize(vb.view(torch.uint8).numpy(), w.kv_scale)
            else:
                kd, vd = kb.to(torch.float64).numpy(), vb.to(torch.float64).numpy()
            K = oracle.gather(kd, table, pos + 1)
            V = oracle.gather(vd, table, pos + 1)
            oracle.attend_two_pass(q.to(torch.float64).numpy(), K, V, w.scale, pos)
            done_units += (pos + 1) * row_kv if w.is_decode else 1
            if time.perf_counter() - t0 > seconds:
                break
    el = time.perf_counter() - t0
    desc = (f"{'requests' if w.is_decode else 'query rows'} of {w.name} drawn at random, "
            f"oracle float64 gather + two-pass softmax, {el:.1f} s wall")
    return done_units, el, desc, threads


# ---------------------------------------------------------------- our arm

def time_prefill_tiles(P, w, t, flush, steps):
    """Device time of the tensor-core tile launch alone on the full GPU: a
    mixed step over only the q_b > 1 requests of the batch (same pools and
    block tables), timed with the library's per-launch events.  In the full
    step the tiles share the GPU with the decode partitions and take fewer
    SMs for longer, so that launch's own duration is not a tile roofline."""
    qsl = w.query_start_loc
    pre = [b for b in range(w.num_seqs) if w.query_lens[b] > 1]
    if not pre:
        return None
    rows = np.concatenate([np.arange(qsl[b], qsl[b + 1]) for b in pre])
    dev = t["q"].device
    q_sub = t["q"][torch.from_numpy(rows).to(dev)].contiguous()
    qlens = w.query_lens[pre]
    qsl_sub = torch.from_numpy(np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)).to(dev)
    lens_sub = torch.from_numpy(w.seq_lens[pre].copy()).to(dev)
    tables_sub = torch.from_numpy(np.ascontiguousarray(w.block_tables[pre])).to(dev)
    out = torch.empty(q_sub.shape, dtype=torch.float32, device=dev)
    nbytes = P.mixed_step_workspace_size(len(pre), q_sub.shape[0], w.num_heads,
                                         tables_sub.shape[1], t["k_cache"])
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)

    def call():
        P.mixed_step(q_sub, t["k_cache"], t["v_cache"], tables_sub, qsl_sub, lens_sub, w.scale,
                     out=out, workspace=ws)
    for _ in range(3):
        call()
    ms = []
    P.kernel_timing(True)
    try:
        for _ in range(min(steps, 50)):
            flush.fill_(1)
            call()
            ms.append(P.kernel_times()["tiles"])
    finally:
        P.kernel_timing(False)
    return statistics.mean(ms), len(ms)


def measure(args, name, rank, world, local, with_e2e=True, with_cpu=True):
    """Time one workload's step on this rank's GPU and return its JSON line
    (every rank computes it; the collectives inside run on every rank)."""
    import paged_kv_cache_434_b200 as P
    from paged_kv_cache_434_b200 import workloads as W

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = workload_for(name, args.seed + rank)
    t = W.make_tensors(w, dev)
    idx = W.index_tensors(w, dev)
    T = w.num_tokens
    decode_only = w.is_decode
    out = torch.empty(T, w.num_heads, w.head_dim, dtype=torch.float32, device=dev)
    slots = torch.empty(T, dtype=torch.int64, device=dev)
    err = P.new_error_word(dev)
    ws_bytes = (P.decode_workspace_size(w.num_seqs, w.num_heads, w.max_blocks_per_seq,
                                        t["k_cache"]) if decode_only else
                P.mixed_step_workspace_size(w.num_seqs, T, w.num_heads, w.max_blocks_per_seq,
                                            t["k_cache"]))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def write():
        # slot mapping and the cache write, one launch
        P.slot_mapping_cache_write(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
                                   idx["block_tables"],
                                   None if decode_only else idx["query_start_loc"],
                                   idx["seq_lens"], slots=slots, err=err, kv_scales=w.kv_scales)

    def attend():
        if decode_only:
            P.decode(t["q"], t["k_cache"], t["v_cache"], idx["block_tables"], idx["seq_lens"],
                     w.scale, out=out, workspace=ws, err=err, kv_scales=w.kv_scales)
        else:
            P.mixed_step(t["q"], t["k_cache"], t["v_cache"], idx["block_tables"],
                         idx["query_start_loc"], idx["seq_lens"], w.scale, out=out,
                         workspace=ws, err=err, kv_scales=w.kv_scales)

    def step():
        if decode_only:  # the write rides in the planner's launch
            P.decode_step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
                          idx["block_tables"], idx["seq_lens"], w.scale, out=out, slots=slots,
                          workspace=ws, err=err, kv_scales=w.kv_scales)
        else:
            write()
            attend()

    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    if P.read_error(err) != 0:
        raise RuntimeError("device error bits set during warm-up")

    # the timed steps carry no event between their launches (an event there
    # would end the launches' programmatic overlap); the attention call alone
    # is timed in a pass of its own below
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    clocks = ClockSampler(dev) if rank == 0 else None
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    wall0 = time.perf_counter()
    for (e0, e2) in evs:
        flush.fill_(1)
        e0.record(stream)
        step()
        e2.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    clk = clocks.stop() if clocks else None
    step_ms = [e0.elapsed_time(e2) for (e0, e2) in evs]
    # the attention call alone: slot mapping and cache write first, untimed
    aevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(min(args.steps, 50))]
    for (e1, e2) in aevs:
        flush.fill_(1)
        write()
        e1.record(stream)
        attend()
        e2.record(stream)
    torch.cuda.synchronize()
    attn_ms = [e1.elapsed_time(e2) for (e1, e2) in aevs]
    total_s = sum(step_ms) / 1e3
    total_s = max_over_ranks(total_s, world, dev)
    if P.read_error(err) != 0:
        raise RuntimeError("device error bits set during the timed steps")

    # ---- per-launch device times: a pass of its own (events between launches
    # end their programmatic overlap, so these steps are not the timed ones)
    n_k = min(args.steps, 50)
    kt = {}
    P.kernel_timing(True)
    try:
        for _ in range(n_k):
            flush.fill_(1)
            step()
            for k, v in P.kernel_times().items():
                kt.setdefault(k, []).append(v)
    finally:
        P.kernel_timing(False)
    kernel_ms = {k: round(statistics.mean(v), 4) for k, v in kt.items()}

    bc = byte_counts(w)
    metric, unit = metric_of(name)
    if name in ("mixed", "mixed_prefill"):
        value = job_throughput(T, args.steps, world, total_s)
    else:
        value = job_throughput(bc["step"], args.steps, world, total_s) / 1e9
    peaks = load_peaks()
    attn_s = statistics.mean(attn_ms) / 1e3
    dominant = "attn_mma_kernel" if w.dtype == "bf16" else "attn_generic_kernel"
    src = "attn_mma.cu" if w.dtype == "bf16" else "attn_common.cu"
    if w.kv_dtype == "fp8":
        extra_kv = {"kv_cache": "e4m3, per-pool scale", "kv_scale": w.kv_scale}
    else:
        extra_kv = {}
    dk_bytes = decode_kernel_bytes(w)
    dk_s = kernel_ms["decode"] / 1e3
    achieved = dk_bytes / dk_s / 1e9
    roofline = {"bound": "hbm", "kernel": dominant,
                "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs, copy)",
                "timed_over": f"the decode-partition launch alone: CUDA events on its stream, "
                              f"mean of {n_k} launches, L2 flushed before each",
                "ms": round(dk_s * 1e3, 4),
                "traffic": kernel_traffic(src, f"{dominant}_{name}.md"),
                "traffic_source": "from profiles/ (ncu summary of the same kernel source)",
                "algorithmic_bytes_per_launch": dk_bytes,
                "attention_call": {"ms": round(attn_s * 1e3, 4),
                                   "achieved": round(bc["attention"] / attn_s / 1e9, 1),
                                   "frac": round(bc["attention"] / attn_s / 1e9 /
                                                 peaks["hbm_gbs"], 4),
                                   "bytes": bc["attention"]}}
    own = own_peaks(dev) if world == 1 else None
    if own is not None and "copy_gbs" in own:
        roofline["own_peaks"] = dict(own, frac_of_own_copy=round(achieved / own["copy_gbs"], 4))
    extra = dict(extra_kv)
    prefill_roofline = None
    if name in ("mixed", "mixed_prefill"):
        fl = prefill_flops(w)
        extra["prefill_flops_per_step"] = fl
        tiles = time_prefill_tiles(P, w, t, flush, args.steps)
        if tiles is not None:
            tiles_ms, n_t = tiles
            tf = fl / (tiles_ms / 1e3) / 1e12
            prefill_roofline = {
                "bound": "tensor", "kernel": "attn_tc_kernel", "achieved": round(tf, 1),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(tf / peaks["bf16_tflops"], 4),
                "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json bf16_tflops, burst: "
                               f"timed alone)",
                "timed_over": f"the tensor-core tile launch on the full GPU: a mixed step over "
                              f"the q_b > 1 requests alone, CUDA events on its stream, mean of "
                              f"{n_t} launches, L2 flushed before each",
                "ms": round(tiles_ms, 4), "algorithmic_flops_per_launch": fl,
                "traffic": kernel_traffic("attn_tc.cu", f"attn_tc_kernel_{name}.md"),
                "traffic_source": "from profiles/ (ncu summary of the same kernel source)"}
            if own is not None and "bf16_gemm_tflops" in own:
                prefill_roofline["frac_of_own_gemm"] = round(tf / own["bf16_gemm_tflops"], 4)

    # ---- end to end: host buffers in, result back to the host, each step.
    # The step's inputs (Q, new K/V, tables, lengths, query offsets) sit in one
    # pinned host buffer and go over in one copy, into one device buffer that
    # the call reads through views; the output comes back in one copy.
    e2e = None
    if with_e2e and not args.no_e2e:
        segs = [(t, n) for n in ("q", "k_new", "v_new")] + \
               [(idx, n) for n in ("block_tables", "seq_lens", "query_start_loc")
                if idx.get(n) is not None]
        offs, tot = [], 0
        for src, n in segs:
            tot = (tot + 255) // 256 * 256  # every view 256-byte aligned
            offs.append(tot)
            tot += src[n].numel() * src[n].element_size()
        host_buf = torch.empty(tot, dtype=torch.uint8).pin_memory()
        dev_buf = torch.empty(tot, dtype=torch.uint8, device=dev)
        saved = [(src, n, src[n]) for src, n in segs]
        for (src, n), off in zip(segs, offs):
            x = src[n]
            nb = x.numel() * x.element_size()
            host_buf[off:off + nb].view(x.dtype).view(x.shape).copy_(x.cpu())
            src[n] = dev_buf[off:off + nb].view(x.dtype).view(x.shape)
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = tot
        d2h = out_h.numel() * out_h.element_size()
        ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        barrier(world)
        torch.cuda.synchronize()
        for (a, b) in ev2:
            flush.fill_(1)
            a.record(stream)
            dev_buf.copy_(host_buf, non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)
            b.record(stream)
        torch.cuda.synchronize()
        for src, n, x in saved:  # the device tensors of the timed steps again
            src[n] = x
        barrier(world)
        e2e_s = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev2) / 1e3, world, dev)
        e2e_val = (T * args.steps * world / e2e_s if name in ("mixed", "mixed_prefill")
                   else bc["step"] * args.steps * world / e2e_s / 1e9)
        e2e = {"value": round(e2e_val, 2), "unit": unit, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_s * 1e3 / args.steps, 4)}

    cpu = None
    if with_cpu and rank == 0 and world == 1 and not args.no_cpu_baseline:
        units, el, desc, threads = oracle_sample(w, (t["k_cache"], t["v_cache"]),
                                                 args.cpu_seconds)
        v = units / el / (1 if name in ("mixed", "mixed_prefill") else 1e9)
        cpu = {"value": round(v, 4), "unit": unit, "cores": threads, "kind": "oracle",
               "sample": desc}

    line = {
        "metric": metric, "value": round(value, 2), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(total_s * 1e3 / args.steps, 4),
        "ms_per_step_p10_p50_p90": [round(float(x), 4) for x in
                                    np.percentile(step_ms, [10, 50, 90])],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("e4m3 pools, f16 tensor-core products" if w.kv_dtype == "fp8" else w.dtype),
        "data": "synthetic: seeded N(0,1) Q/K/V rounded to the dtype, seeded lengths and "
                "randomly permuted physical blocks",
        "config": {"workload": w.name, "num_seqs": w.num_seqs, "num_tokens": T,
                   "num_heads": w.num_heads, "num_kv_heads": w.num_kv_heads,
                   "head_dim": w.head_dim, "block_size": w.block_size,
                   "num_blocks": w.num_blocks,
                   "kv_bytes_unique": bc["kv"], "step_bytes": bc["step"],
                   "l2": L2_NOTE,
                   "parallelism": f"replicas x{world} (independent batches per GPU)",
                   **extra},
        "roofline": roofline,
        **({"prefill_roofline": prefill_roofline} if prefill_roofline else {}),
        "cpu_baseline": cpu,
        "e2e": e2e,
        "kernel_ms": kernel_ms,
        # a decode step's write is in the planner's launch; a mixed step's is its own
        "gpu_launches": (len(kernel_ms) + (0 if decode_only else 1)) * args.steps,
        "clocks": clk,
        "wall_s_timed_region": round(wall, 3),
    }
    if unit == "tokens/s":
        # the same metric without the slot mapping and cache write: query tokens
        # over the attention call alone (planner, tiles, partitions, merge), from
        # the per-launch timing pass
        line["without_cache_write"] = {
            "value": round(T * world / attn_s, 2), "unit": "tokens/s",
            "ms": round(attn_s * 1e3, 4),
            "timed_over": "the attention call alone, CUDA events on its stream in the "
                          "per-launch timing pass"}
    return line


def _in_step_tiles(line):
    """The tensor-core tile launch of the full mixed step, on the SMs the
    planner gave it (per-launch timing pass), as a fraction of the bf16 peak."""
    fl = line["config"].get("prefill_flops_per_step")
    ms = line["kernel_ms"].get("tiles")
    if not fl or not ms:
        return None
    peaks = load_peaks()
    tf = fl / (ms / 1e3) / 1e12
    return {"bound": "tensor", "kernel": "attn_tc_kernel", "achieved": round(tf, 1),
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(tf / peaks["bf16_tflops"], 4), "ms": ms,
            "timed_over": "the tile launch inside the full mixed step, on the SMs the planner "
                          "leaves to the tiles (the decode partitions run on the others); CUDA "
                          "events on its stream in the per-launch timing pass"}


def run_ours(args, rank, world, local):
    line = measure(args, args.workload, rank, world, local)
    if args.workload == "llama8b_decode" and not args.no_extras:
        # The other half of the metric (a mixed continuous-batching step), the
        # shared-prefix decode batch and the long-context split-KV batch,
        # measured in the same process after the headline, each with its own
        # timed region, clocks and launch count.
        torch.cuda.empty_cache()
        m = measure(args, "mixed", rank, world, local, with_cpu=False)
        line["mixed_step"] = {
            k: m[k] for k in ("metric", "value", "unit", "ms_per_step", "without_cache_write",
                              "e2e", "kernel_ms", "gpu_launches", "clocks") if k in m}
        line["mixed_step"]["config"] = {k: m["config"][k] for k in (
            "workload", "num_seqs", "num_tokens", "prefill_flops_per_step")}
        line["mixed_step"]["prefill_roofline"] = {"alone": m.get("prefill_roofline"),
                                                  "in_step": _in_step_tiles(m)}
        line["mixed_step"]["decode_roofline"] = m["roofline"]
        torch.cuda.empty_cache()
        sp = measure(args, "shared_prefix", rank, world, local, with_cpu=False)
        line["shared_prefix"] = {
            k: sp[k] for k in ("metric", "value", "unit", "ms_per_step", "e2e", "kernel_ms",
                               "gpu_launches", "clocks")}
        line["shared_prefix"]["config"] = {k: sp["config"][k] for k in (
            "workload", "num_seqs", "num_heads", "num_kv_heads", "block_size",
            "kv_bytes_unique")}
        line["shared_prefix"]["attention_call"] = dict(
            sp["roofline"]["attention_call"],
            note="per attention call, on unique bytes: each physical block once (the shared "
                 "prefix once), Q read and fp32 O written, against the HBM copy peak")
        line["shared_prefix"]["suffix_partitions"] = sp["roofline"]
        torch.cuda.empty_cache()
        lc = measure(args, "long_context", rank, world, local, with_cpu=False)
        line["long_context"] = {
            k: lc[k] for k in ("metric", "value", "unit", "ms_per_step", "e2e", "kernel_ms",
                               "gpu_launches", "clocks", "roofline")}
        line["long_context"]["config"] = {k: lc["config"][k] for k in (
            "workload", "num_seqs", "num_heads", "num_kv_heads", "block_size",
            "kv_bytes_unique")}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- reference arm

# ---------------------------------------------------------------- fused RoPE + cache write

ROPE_THETA = 500000.0


def rope_inputs(w, dev, seed):
    """New tokens of the step: q/k/v rows, positions, a pool with just room for
    them (randomly permuted slots, so the scatter is as irregular as a real
    pool's) and the slot of every token."""
    rng = np.random.default_rng([seed, 79])
    T, hq, hkv, d = w.num_tokens, w.num_heads, w.num_kv_heads, w.head_dim
    pos = np.concatenate([np.arange(w.seq_lens[b] - w.query_lens[b], w.seq_lens[b])
                          for b in range(w.num_seqs)]).astype(np.int64)
    nb = (T + w.block_size - 1) // w.block_size + 64
    slots = rng.permutation(nb * w.block_size)[:T].astype(np.int64)
    g = torch.Generator(device=dev).manual_seed(seed)
    mk = lambda *sh: torch.randn(*sh, generator=g, device=dev).to(torch.bfloat16)
    return {"q": mk(T, hq, d), "k": mk(T, hkv, d), "v": mk(T, hkv, d),
            "k_cache": torch.zeros(nb, w.block_size, hkv, d, dtype=torch.bfloat16, device=dev),
            "v_cache": torch.zeros(nb, w.block_size, hkv, d, dtype=torch.bfloat16, device=dev),
            "positions": torch.from_numpy(pos).to(dev), "slots": torch.from_numpy(slots).to(dev),
            "max_pos": int(pos.max()) + 1}


def rope_bytes(w):
    """Algorithmic bytes of the fused launch: Q read and written, K and V read
    and written to the pools, one float32 table row, the position and the slot
    per token."""
    T, e = w.num_tokens, w.elt_bytes
    return T * (2 * w.num_heads * w.head_dim * e + 4 * w.num_kv_heads * w.head_dim * e +
                w.head_dim * 4 + 16)


def run_rope(args, rank, world, local):
    import paged_kv_cache_434_b200 as P
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = workload_for("rope_write", args.seed + rank)
    x = rope_inputs(w, dev, args.seed + rank)
    table = P.rope_cos_sin_cache(x["max_pos"], w.head_dim, ROPE_THETA, device=dev)
    q_out = torch.empty_like(x["q"])
    err = P.new_error_word(dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def step():
        P.rope_cache_write(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], x["slots"],
                           x["positions"], table, neox=True, q_out=q_out, err=err)

    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    if P.read_error(err) != 0:
        raise RuntimeError("device error bits set during warm-up")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    clocks = ClockSampler(dev) if rank == 0 else None
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    wall0 = time.perf_counter()
    for a, b in evs:
        flush.fill_(1)
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    clk = clocks.stop() if clocks else None
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_s = max_over_ranks(sum(step_ms) / 1e3, world, dev)
    nbytes = rope_bytes(w)
    value = nbytes * args.steps * world / total_s / 1e9
    peaks = load_peaks()
    k_s = statistics.mean(step_ms) / 1e3        # one launch per step: the kernel's own time
    achieved = nbytes / k_s / 1e9
    roofline = {"bound": "hbm", "kernel": "rope_cache_write_kernel", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs, copy)",
                "timed_over": f"the fused launch (the step's only launch): CUDA events on its "
                              f"stream, mean of {args.steps} launches, L2 flushed before each",
                "ms": round(k_s * 1e3, 4),
                "traffic": kernel_traffic("rope.cu", "rope_cache_write_kernel_rope_write.md"),
                "algorithmic_bytes_per_launch": nbytes}
    e2e = None
    if not args.no_e2e:
        host = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "positions", "slots")}
        out_h = torch.empty(q_out.shape, dtype=q_out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = out_h.numel() * out_h.element_size()
        ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        torch.cuda.synchronize()
        for a, b in ev2:
            flush.fill_(1)
            a.record(stream)
            for n, t in host.items():
                x[n].copy_(t, non_blocking=True)
            step()
            out_h.copy_(q_out, non_blocking=True)
            b.record(stream)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev2) / 1e3, world, dev)
        e2e = {"value": round(nbytes * args.steps * world / e2e_s / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e2e_s * 1e3 / args.steps, 4)}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = rope_oracle_sample(w, x, args.cpu_seconds)
    if rank == 0:
        print(json.dumps({
            "metric": "fused RoPE + cache write GB/s", "value": round(value, 2), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
            "ms_per_step": round(total_s * 1e3 / args.steps, 4),
            "ms_per_step_p10_p50_p90": [round(float(v), 4) for v in
                                        np.percentile(step_ms, [10, 50, 90])],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) Q/K/V rounded to bf16, the mixed step's positions, "
                    "randomly permuted slots",
            "config": {"workload": "rope_cache_write_llama3_8b_8192_tokens", "num_tokens": w.num_tokens,
                       "num_heads": w.num_heads, "num_kv_heads": w.num_kv_heads,
                       "head_dim": w.head_dim, "rotary_dim": w.head_dim, "rope_theta": ROPE_THETA,
                       "pairing": "split-half (neox)", "step_bytes": nbytes,
                       "l2": L2_NOTE,
                       "parallelism": f"replicas x{world} (independent batches per GPU)"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps, "clocks": clk, "wall_s_timed_region": round(wall, 3)}),
            flush=True)


def rope_oracle_sample(w, x, seconds, rng_seed=0):
    """The oracle's fused step on whole tokens until `seconds` pass (bytes/s
    of the same algorithmic count)."""
    import oracle
    rng = np.random.default_rng(rng_seed)
    table = oracle.cos_sin_table(x["max_pos"], w.head_dim, ROPE_THETA)
    T = w.num_tokens
    order = rng.permutation(T)[:2048]
    q = x["q"][torch.from_numpy(order).to(x["q"].device)].cpu().to(torch.float64).numpy()
    k = x["k"][torch.from_numpy(order).to(x["q"].device)].cpu().to(torch.float64).numpy()
    v = x["v"][torch.from_numpy(order).to(x["q"].device)].cpu().to(torch.float64).numpy()
    pos = x["positions"].cpu().numpy()[order]
    nb = 64
    kp = np.zeros((nb, w.block_size, w.num_kv_heads, w.head_dim))
    vp = np.zeros_like(kp)
    slots = np.arange(len(order)) % (nb * w.block_size)
    done, t0 = 0, time.perf_counter()
    for i in range(0, len(order), 64):
        sl = slice(i, i + 64)
        oracle.rope_cache_write(q[sl], k[sl], v[sl], pos[sl], slots[sl], kp, vp, table,
                                w.head_dim, True)
        done += min(64, len(order) - i)
        if time.perf_counter() - t0 > seconds:
            break
    el = time.perf_counter() - t0
    per_tok = rope_bytes(w) / T
    return {"value": round(done * per_tok / el / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{done} of the {T} tokens (64 per call), float64 NumPy, one thread"}


def run_reference(args, rank, world, local):
    """The CPU oracle timed as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    import paged_kv_cache_434_b200.workloads as W
    w = workload_for(args.workload, args.seed)
    metric, unit = metric_of(args.workload)
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    pools = None
    if dev.type == "cuda":
        t = W.make_tensors(w, dev)
        pools = (t["k_cache"], t["v_cache"])
    else:
        t = W.make_tensors(w, "cpu", where="host")
        pools = (t["k_cache"], t["v_cache"])
    per_step = max(0.1, min(args.cpu_seconds, 60.0 / max(1, args.steps + args.warmup)))
    vals = []
    desc = threads = None
    for k in range(max(args.warmup, 3) + args.steps):
        units, el, desc, threads = oracle_sample(w, pools, per_step, rng_seed=k)
        if k >= max(args.warmup, 3):
            vals.append((units, el))
    units = sum(u for u, _ in vals)
    el = sum(e for _, e in vals)
    value = units / el / (1 if args.workload in ("mixed", "mixed_prefill") else 1e9)
    line = {
        "impl": "reference", "metric": metric, "value": round(value, 4), "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(el * 1e3 / max(1, args.steps), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same generator and seed as our arm)",
        "config": {"workload": w.name},
        "cpu_baseline": {"value": round(value, 4), "unit": unit, "cores": threads,
                         "kind": "oracle", "sample": f"each step: {desc}"},
        "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- copy-on-write block copies

COW_BLOCKS, COW_PAIRS = 8192, 2048


def cow_inputs(dev, seed):
    g = torch.Generator(device=dev).manual_seed(seed)
    mk = lambda: torch.randn(COW_BLOCKS, 16, 8, 128, generator=g, device=dev).to(torch.bfloat16)
    ids = np.random.default_rng([seed, 81]).permutation(COW_BLOCKS)
    m = np.stack([ids[:COW_PAIRS], ids[COW_PAIRS:2 * COW_PAIRS]], axis=1).astype(np.int64)
    return mk(), mk(), torch.from_numpy(m).to(dev)


def cow_bytes():
    return COW_PAIRS * 2 * 2 * (16 * 8 * 128 * 2)   # pairs x pools x (read + write) x block


def cow_oracle_sample(kc, vc, seconds):
    """The oracle's block copy (NumPy, one thread) on 512 pairs per call in
    1024-block pools cut from the same data, for `seconds`."""
    import oracle
    kh = kc[:1024].cpu().view(torch.int16).numpy()
    vh = vc[:1024].cpu().view(torch.int16).numpy()
    pairs = np.stack([np.arange(0, 512), np.arange(512, 1024)], axis=1)
    done, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        oracle.copy_blocks(kh, vh, pairs)
        done += len(pairs)
    el = time.perf_counter() - t0
    return {"value": round(done * cow_bytes() / COW_PAIRS / el / 1e9, 4), "unit": "GB/s",
            "cores": 1, "kind": "oracle",
            "sample": f"{done} block pairs (512 per call) in 1024-block pools, NumPy, one thread"}


def run_cow_reference(args, rank, world, local):
    """The oracle's block copy timed as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    kc, vc, _ = cow_inputs(dev, args.seed)
    warm = max(args.warmup, 3)
    per = max(0.5, min(args.cpu_seconds, 60.0 / max(1, args.steps)))
    for _ in range(warm):
        cow_oracle_sample(kc, vc, 0.1)
    vals = [cow_oracle_sample(kc, vc, per)["value"] for _ in range(args.steps)]
    v = statistics.mean(vals)
    print(json.dumps({
        "impl": "reference", "metric": "copy-on-write block copy GB/s",
        "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": warm,
        "ms_per_step": round(cow_bytes() / (v * 1e9) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 bits", "data": "synthetic (same generator and seed as our arm)",
        "config": {"workload": "cow_copy_llama3_8b_2048_pairs"},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": 1,
                         "kind": "oracle",
                         "sample": f"each step: about {per:.1f} s of 512-pair copies"},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0}), flush=True)


def run_cow(args, rank, world, local):
    import paged_kv_cache_434_b200 as P
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kc, vc, m = cow_inputs(dev, args.seed + rank)
    err = P.new_error_word(dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()
    step = lambda: P.copy_blocks(kc, vc, m, err=err)
    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    if P.read_error(err) != 0:
        raise RuntimeError("device error bits set during warm-up")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    clocks = ClockSampler(dev) if rank == 0 else None
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    wall0 = time.perf_counter()
    for a, b in evs:
        flush.fill_(1)
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    clk = clocks.stop() if clocks else None
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_s = max_over_ranks(sum(step_ms) / 1e3, world, dev)
    nbytes = cow_bytes()
    value = nbytes * args.steps * world / total_s / 1e9
    peaks = load_peaks()
    k_s = statistics.mean(step_ms) / 1e3
    achieved = nbytes / k_s / 1e9
    e2e = None
    if not args.no_e2e:
        # end to end: the pair list comes from the host each step (the pools
        # stay on the device: a copy-on-write never moves them)
        m_h = m.cpu().pin_memory()
        chk = torch.empty(COW_PAIRS, 16, 8, 128, dtype=torch.bfloat16).pin_memory()
        ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        torch.cuda.synchronize()
        for a, b in ev2:
            flush.fill_(1)
            a.record(stream)
            m.copy_(m_h, non_blocking=True)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev2) / 1e3, world, dev)
        e2e = {"value": round(nbytes * args.steps * world / e2e_s / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": m_h.numel() * 8, "d2h_bytes_per_step": 0,
               "ms_per_step": round(e2e_s * 1e3 / args.steps, 4),
               "note": "the step's result stays in the device pools; nothing is read back"}
        del chk
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cow_oracle_sample(kc, vc, min(args.cpu_seconds, 5.0))
    if rank == 0:
        print(json.dumps({
            "metric": "copy-on-write block copy GB/s", "value": round(value, 2), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
            "ms_per_step": round(total_s * 1e3 / args.steps, 4),
            "ms_per_step_p10_p50_p90": [round(float(v), 4) for v in
                                        np.percentile(step_ms, [10, 50, 90])],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) pools, random disjoint source/destination blocks",
            "config": {"workload": "cow_copy_llama3_8b_2048_pairs", "pairs": COW_PAIRS,
                       "num_blocks": COW_BLOCKS, "block_size": 16, "num_kv_heads": 8,
                       "head_dim": 128, "step_bytes": nbytes,
                       "l2": L2_NOTE,
                       "parallelism": f"replicas x{world} (independent pools per GPU)"},
            "roofline": {"bound": "hbm", "kernel": "copy_blocks_kernel", "achieved": round(achieved, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4),
                         "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs, copy)",
                         "timed_over": f"the copy launch (the step's only launch): CUDA events on "
                                       f"its stream, mean of {args.steps} launches",
                         "ms": round(k_s * 1e3, 4),
                         "traffic": kernel_traffic("blocks.cu", "copy_blocks_kernel_cow_copy.md"),
                         "algorithmic_bytes_per_launch": nbytes},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps, "clocks": clk,
            "wall_s_timed_region": round(wall, 3)}), flush=True)


# ---------------------------------------------------------------- CUDA graph decode step

GRAPH_LENS = [512, 1024, 1536, 2048]


def run_graph(args, rank, world, local):
    import paged_kv_cache_434_b200 as P
    from paged_kv_cache_434_b200 import workloads as W
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = W.custom("graph_decode_llama3_8b_b4", GRAPH_LENS, [1] * len(GRAPH_LENS), 32, 8, 128, 16,
                 "bf16", seed=args.seed + rank)
    t = W.make_tensors(w, dev)
    idx = W.index_tensors(w, dev)
    T = w.num_tokens
    ws = torch.empty(P.decode_workspace_size(w.num_seqs, w.num_heads, w.max_blocks_per_seq,
                                             t["k_cache"]), dtype=torch.uint8, device=dev)
    slots = torch.empty(T, dtype=torch.int64, device=dev)
    out = torch.empty(T, w.num_heads, w.head_dim, dtype=torch.float32, device=dev)
    err = P.new_error_word(dev)
    flush = L2Flush(dev)

    def step():
        P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
               idx["query_start_loc"], idx["seq_lens"], w.scale, decode_only=True, out=out,
               slots=slots, workspace=ws, err=err)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        step()
    for _ in range(max(args.warmup, 3)):
        g.replay()
    torch.cuda.synchronize()
    if P.read_error(err) != 0:
        raise RuntimeError("device error bits set during warm-up")
    stream = torch.cuda.current_stream()

    def timed(fn, flush_l2):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        torch.cuda.synchronize()
        for a, b in evs:
            if flush_l2:
                flush.fill_(1)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    clocks = ClockSampler(dev) if rank == 0 else None
    barrier(world)
    if clocks:
        clocks.start()
    wall0 = time.perf_counter()
    g_ms = timed(g.replay, True)
    wall = time.perf_counter() - wall0
    clk = clocks.stop() if clocks else None
    e_ms = timed(step, True)
    g_hot = timed(g.replay, False)      # back to back, L2 warm: the launch-bound regime
    e_hot = timed(step, False)
    total_s = max_over_ranks(sum(g_ms) / 1e3, world, dev)
    bc = byte_counts(w)
    us = total_s * 1e6 / args.steps
    e2e = None
    if not args.no_e2e:
        names = ["q", "k_new", "v_new"]
        host = {n: t[n].cpu().pin_memory() for n in names}
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in host.values())
        ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        torch.cuda.synchronize()
        for a, b in ev2:
            flush.fill_(1)
            a.record(stream)
            for n in names:
                t[n].copy_(host[n], non_blocking=True)
            g.replay()
            out_h.copy_(out, non_blocking=True)
            b.record(stream)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev2) / 1e3, world, dev)
        e2e = {"value": round(e2e_s * 1e6 / args.steps, 2), "unit": "us/step",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": out_h.numel() * 4}
    peaks = load_peaks()
    achieved = bc["step"] / (statistics.mean(g_ms) / 1e3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "decode step us (CUDA graph replay)", "value": round(us, 2),
            "unit": "us/step", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": round(us / 1e3, 5),
            "ms_per_step_p10_p50_p90": [round(float(v), 5) for v in np.percentile(g_ms, [10, 50, 90])],
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) Q/K/V rounded to bf16, permuted physical blocks",
            "config": {"workload": w.name, "num_seqs": w.num_seqs, "seq_lens": GRAPH_LENS,
                       "num_heads": 32, "num_kv_heads": 8, "head_dim": 128, "block_size": 16,
                       "step_bytes": bc["step"],
                       "l2": L2_NOTE,
                       "parallelism": f"replicas x{world}"},
            "eager_us_per_step": round(statistics.mean(e_ms) * 1e3, 2),
            "l2_warm_back_to_back_us": {"graph": round(statistics.mean(g_hot) * 1e3, 2),
                                        "eager": round(statistics.mean(e_hot) * 1e3, 2)},
            "roofline": {"bound": "hbm", "kernel": "the whole step (graph replay)",
                         "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4),
                         "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs, copy)",
                         "timed_over": "one replay per step, CUDA events on the stream",
                         "traffic": None, "algorithmic_bytes_per_launch": bc["step"],
                         "note": f"{bc['step'] / 1e6:.0f} MB per step: launch- and "
                                 f"latency-bound, not an HBM roofline"},
            "cpu_baseline": None, "e2e": e2e, "gpu_launches": 3 * args.steps, "clocks": clk,
            "wall_s_timed_region": round(wall, 3)}), flush=True)
    del g


def run_rope_reference(args, rank, world, local):
    """The oracle's fused RoPE + cache write timed as the reference arm."""
    if rank != 0:
        return
    w = workload_for("rope_write", args.seed)
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    if dev.type == "cuda":
        x = rope_inputs(w, dev, args.seed)
    else:
        x = rope_inputs_cpu(w, args.seed)
    per_step = max(0.1, min(args.cpu_seconds, 60.0 / max(1, args.steps + args.warmup)))
    vals = [rope_oracle_sample(w, x, per_step, rng_seed=k)["value"]
            for k in range(max(args.warmup, 3) + args.steps)][max(args.warmup, 3):]
    value = statistics.mean(vals)
    print(json.dumps({
        "impl": "reference", "metric": "fused RoPE + cache write GB/s", "value": round(value, 4),
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(rope_bytes(w) / (value * 1e9) * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same generator and seed as our arm)",
        "config": {"workload": "rope_cache_write_llama3_8b_8192_tokens"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: about {per_step:.1f} s of whole tokens"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0}), flush=True)


def rope_inputs_cpu(w, seed):
    rng = np.random.default_rng([seed, 80])
    T, hq, hkv, d = w.num_tokens, w.num_heads, w.num_kv_heads, w.head_dim
    pos = np.concatenate([np.arange(w.seq_lens[b] - w.query_lens[b], w.seq_lens[b])
                          for b in range(w.num_seqs)]).astype(np.int64)
    mk = lambda *sh: torch.from_numpy(rng.standard_normal(sh, dtype=np.float32)).to(torch.bfloat16)
    return {"q": mk(T, hq, d), "k": mk(T, hkv, d), "v": mk(T, hkv, d),
            "positions": torch.from_numpy(pos), "max_pos": int(pos.max()) + 1}


def main():
    args = parse_args()
    rank, world, local = dist_setup()
    try:
        if args.workload == "graph_decode":
            if args.impl == "reference":
                if rank == 0:
                    print(json.dumps({"impl": "reference", "unavailable":
                                      "a CUDA graph step has no CPU counterpart; the oracle is "
                                      "timed on the decode workloads"}), flush=True)
            else:
                run_graph(args, rank, world, local)
        elif args.workload == "cow_copy":
            if args.impl == "reference":
                run_cow_reference(args, rank, world, local)
            else:
                run_cow(args, rank, world, local)
        elif args.workload == "rope_write":
            if args.impl == "reference":
                run_rope_reference(args, rank, world, local)
            else:
                run_rope(args, rank, world, local)
        elif args.impl == "reference":
            run_reference(args, rank, world, local)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

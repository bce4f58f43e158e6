"""A decode step (slot mapping -> cache write -> attention) captured in a CUDA
graph: every launch of the step is capture-safe (no host synchronisation, no
allocation, tensor maps passed by value), replays give the same bits as
eager calls, and a replay after the inputs change in place follows them."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_434_b200 as P
from paged_kv_cache_434_b200 import workloads as W
from _util import assert_close, bits, f64, oracle_full

pytestmark = pytest.mark.gpu


def _decode_case(seed, lens, dtype="bf16"):
    w = W.custom(f"graph_{seed}", lens, [1] * len(lens), 32, 8, 128, 16, dtype, seed=seed,
                 extra_blocks=8)
    host = W.make_tensors(w, "cpu", where="host")
    return w, host


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_graph_replay_matches_eager(cuda_device, dtype):
    dev = cuda_device
    w, host = _decode_case(3, [700, 33, 1500, 256], dtype)
    idx = W.index_tensors(w, dev)
    T = w.num_tokens
    ws = torch.empty(P.decode_workspace_size(w.num_seqs, w.num_heads, w.max_blocks_per_seq,
                                             host["k_cache"]), dtype=torch.uint8, device=dev)
    slots = torch.empty(T, dtype=torch.int64, device=dev)
    err = P.new_error_word(dev)

    def fresh():
        return {k: v.to(dev) for k, v in host.items()}

    # eager reference
    t = fresh()
    out_e = torch.empty(T, w.num_heads, w.head_dim, dtype=torch.float32, device=dev)
    P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
           idx["query_start_loc"], idx["seq_lens"], w.scale, decode_only=True, out=out_e,
           slots=slots, workspace=ws, err=err)
    torch.cuda.synchronize()
    eager = out_e.cpu()
    # capture the same step on fresh pools, replay twice
    t = fresh()
    out_g = torch.empty_like(out_e)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        P.step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], idx["block_tables"],
               idx["query_start_loc"], idx["seq_lens"], w.scale, decode_only=True, out=out_g,
               slots=slots, workspace=ws, err=err)
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(bits(out_g.cpu()), bits(eager))
    g.replay()                          # the same write again: same cache, same output
    torch.cuda.synchronize()
    assert np.array_equal(bits(out_g.cpu()), bits(eager))
    # new queries / new tokens written in place: the replay follows them
    rng = np.random.default_rng(9)
    td = t["q"].dtype
    q2 = torch.from_numpy(rng.standard_normal(tuple(t["q"].shape), dtype=np.float32)).to(td)
    k2 = torch.from_numpy(rng.standard_normal(tuple(t["k_new"].shape), dtype=np.float32)).to(td)
    t["q"].copy_(q2)
    t["k_new"].copy_(k2)
    g.replay()
    torch.cuda.synchronize()
    assert P.read_error(err) == 0
    host2 = dict(host)
    host2["q"], host2["k_new"] = q2, k2
    _, _, _, ref, _, valid = oracle_full(w, host2)
    assert_close(f64(out_g.cpu())[valid], ref[valid], w.dtype, "graph replay, new inputs")
    del g

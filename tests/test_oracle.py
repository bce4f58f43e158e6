"""Pins for the CPU oracle (no GPU).

Each test ties an oracle function to something other than itself: the worked
slot example printed on the page, a closed form, brute force, a library
attention routine (torch SDPA in float64), or an invariant.  The last group
plants plausible mistakes in a copy of the oracle and checks that at least
one pin catches each of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oatt

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- slot mapping

def test_slot_worked_example():
    g = _golden("slot_worked_example.json")
    assert oracle.slot_of(g["block_table"], g["position"], g["block_size"]) == g["slot"]
    # the intermediate quantities the page prints
    assert g["position"] // g["block_size"] == g["logical_block"]
    assert g["block_table"][g["logical_block"]] == g["physical_block"]
    assert g["position"] % g["block_size"] == g["block_offset"]


def test_slot_worked_example_through_slot_mapping():
    g = _golden("slot_worked_example.json")
    table = np.array([g["block_table"]], dtype=np.int32)
    # request 0 of length 26 with its last token (position 25) new this step
    slots = oracle.slot_mapping(table, [0, 1], [g["position"] + 1], g["block_size"])
    assert slots.tolist() == [g["slot"]]


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_slot_mapping_is_a_bijection_onto_the_pool(bs):
    nb = 16
    order = np.random.default_rng(7).permutation(nb).astype(np.int32)
    table = order[None, :]
    L = nb * bs
    slots = oracle.slot_mapping(table, [0, L], [L], bs)
    assert sorted(slots.tolist()) == list(range(nb * bs))
    # round trip: slot -> (slot // bs, slot % bs) recovers (table[p // bs], p % bs)
    for p, s in enumerate(slots):
        assert (s // bs, s % bs) == (order[p // bs], p % bs)


def test_slot_mapping_only_new_tokens_at_the_end():
    table = np.array([[3, 1, -1], [0, 2, 4]], dtype=np.int32)
    # request 0: 20 tokens, 3 new (positions 17,18,19); request 1: 33 tokens, 1 new (32)
    slots = oracle.slot_mapping(table, [0, 3, 4], [20, 33], 16)
    assert slots.tolist() == [1 * 16 + 1, 1 * 16 + 2, 1 * 16 + 3, 4 * 16 + 0]


# ---------------------------------------------------------------- cache write

def test_cache_write_every_slot_once_random_order():
    nb, bs, hkv, d = 4, 16, 2, 8
    n = nb * bs
    slots = np.random.default_rng(3).permutation(n).astype(np.int64)
    # token t's row is filled with the value t, so the pool shows which token landed where
    k = np.broadcast_to(np.arange(n, dtype=np.float32)[:, None, None], (n, hkv, d)).copy()
    v = -k
    kc = np.full((nb, bs, hkv, d), np.nan, dtype=np.float32)
    vc = kc.copy()
    k2, v2, err = oracle.cache_write(kc, vc, k, v, slots)
    assert err == set()
    flat_k = k2.reshape(nb * bs, hkv, d)  # row-major: flat row = block * bs + offset
    flat_v = v2.reshape(nb * bs, hkv, d)
    for t, s in enumerate(slots):
        assert np.all(flat_k[s] == t) and np.all(flat_v[s] == -t)


def test_cache_write_is_bit_exact_on_raw_bf16_bits():
    rng = np.random.default_rng(5)
    nb, bs, hkv, d = 3, 8, 2, 16
    bits = rng.integers(0, 1 << 16, size=(nb, bs, hkv, d), dtype=np.uint16)
    new = rng.integers(0, 1 << 16, size=(2, hkv, d), dtype=np.uint16)
    k2, _, err = oracle.cache_write(bits, bits, new, new, [5, 17])
    assert err == set()
    assert np.array_equal(k2[0, 5], new[0]) and np.array_equal(k2[2, 1], new[1])
    mask = np.ones((nb, bs), bool)
    mask[0, 5] = mask[2, 1] = False
    assert np.array_equal(k2[mask], bits[mask])


def test_cache_write_padding_and_out_of_range():
    nb, bs = 2, 4
    kc = np.zeros((nb, bs, 1, 2))
    k = np.ones((3, 1, 2))
    k2, _, err = oracle.cache_write(kc, kc, k, k, [-1, nb * bs, 3])
    assert err == {oracle.ERR_SLOT_OOB}
    assert k2.sum() == 2 and np.all(k2[0, 3] == 1)


def test_gather_follows_the_block_table():
    nb, bs = 5, 4
    cache = np.arange(nb * bs, dtype=np.float64).reshape(nb, bs, 1, 1)
    K = oracle.gather(cache, [3, 0, 4], 10)
    assert K[:, 0, 0].tolist() == [12, 13, 14, 15, 0, 1, 2, 3, 16, 17]


# ---------------------------------------------------------------- attention

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa_reference(q, K, V, scale, first_pos):
    """torch scaled_dot_product_attention in float64 with an explicit boolean
    mask (bottom-right causal) and K/V expanded to the query heads."""
    n_q, hq, d = q.shape
    L, hkv, _ = K.shape
    g = hq // hkv
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                         # [1,Hq,n_q,D]
    kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(g, 0)[None]  # [1,Hq,L,D]
    vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(g, 0)[None]
    mask = torch.arange(L)[None, :] <= (first_pos + torch.arange(n_q))[:, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


CASES = [
    # n_q, Hq, Hkv, D, L
    (1, 8, 2, 64, 40),
    (1, 4, 4, 16, 1),
    (5, 6, 3, 8, 37),
    (17, 8, 1, 32, 50),
    (33, 4, 2, 16, 33),
]


@pytest.mark.parametrize("case", CASES)
def test_two_pass_matches_library_sdpa(case):
    n_q, hq, hkv, d, L = case
    q, K, V = _rand((n_q, hq, d), 1), _rand((L, hkv, d), 2), _rand((L, hkv, d), 3)
    scale = 1 / math.sqrt(d)
    ref = _sdpa_reference(q, K, V, scale, L - n_q)
    got = oracle.attend_two_pass(q, K, V, scale, L - n_q)
    assert np.max(np.abs(got - ref)) < 1e-12


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("tile", [1, 7, 16])
def test_online_softmax_equals_two_pass(case, tile):
    n_q, hq, hkv, d, L = case
    q, K, V = _rand((n_q, hq, d), 4), _rand((L, hkv, d), 5), _rand((L, hkv, d), 6)
    a = oracle.attend_two_pass(q, K, V, 0.3, L - n_q)
    b = oracle.attend_online(q, K, V, 0.3, L - n_q, tile=tile)
    assert np.max(np.abs(a - b)) < 1e-12


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("parts", [1, 2, 7])
def test_split_kv_merge_equals_unsplit(case, parts):
    n_q, hq, hkv, d, L = case
    q, K, V = _rand((n_q, hq, d), 7), _rand((L, hkv, d), 8), _rand((L, hkv, d), 9)
    a = oracle.attend_two_pass(q, K, V, 0.2, L - n_q)
    b = oracle.attend_split(q, K, V, 0.2, L - n_q, parts)
    assert np.max(np.abs(a - b)) < 1e-12


@pytest.mark.parametrize("case", [(1, 4, 2, 4, 5), (3, 2, 1, 3, 6), (2, 4, 4, 2, 3)])
def test_brute_force_agrees(case):
    n_q, hq, hkv, d, L = case
    q, K, V = _rand((n_q, hq, d), 10), _rand((L, hkv, d), 11), _rand((L, hkv, d), 12)
    a = oracle.attend_two_pass(q, K, V, 0.7, L - n_q)
    b = np.array(oracle.brute_attention(q.tolist(), K.tolist(), V.tolist(), 0.7, L - n_q))
    assert np.max(np.abs(a - b)) < 1e-12


def test_context_length_one_returns_v_exactly():
    q, K, V = _rand((1, 8, 64), 13), _rand((1, 2, 64), 14), _rand((1, 2, 64), 15)
    out = oracle.attend_two_pass(q, K, V, 0.125, 0)
    for h in range(8):
        assert np.array_equal(out[0, h], V[0, h // 4])


def test_identical_keys_return_mean_of_v():
    L = 23
    K = np.repeat(_rand((1, 2, 16), 16), L, axis=0)
    V = _rand((L, 2, 16), 17)
    out = oracle.attend_two_pass(_rand((1, 4, 16), 18), K, V, 0.25, L - 1)
    for h in range(4):
        assert np.max(np.abs(out[0, h] - V[:, h // 2].mean(axis=0))) < 1e-14


def test_chunk_after_prefix_equals_rows_of_full_prefill():
    L, n_q, hq, hkv, d = 29, 9, 4, 2, 8
    q_full, K, V = _rand((L, hq, d), 19), _rand((L, hkv, d), 20), _rand((L, hkv, d), 21)
    full = oracle.attend_two_pass(q_full, K, V, 0.5, 0)
    chunk = oracle.attend_two_pass(q_full[L - n_q:], K, V, 0.5, L - n_q)
    assert np.max(np.abs(full[L - n_q:] - chunk)) < 1e-13


def test_first_query_of_fresh_prompt_returns_v0():
    L, hq, hkv, d = 12, 4, 2, 8
    q, K, V = _rand((L, hq, d), 22), _rand((L, hkv, d), 23), _rand((L, hkv, d), 24)
    out = oracle.attend_two_pass(q, K, V, 0.5, 0)
    for h in range(hq):
        assert np.array_equal(out[0, h], V[0, h // 2])


def test_kv_cache_size_closed_form():
    g = _golden("llama3_8b_kv_size.json")
    got = oracle.kv_cache_bytes(g["num_layers"], g["num_kv_heads"], g["head_dim"],
                                g["bytes_per_elt"], g["context_len"])
    assert got == g["kv_bytes"] == 2 ** 30


# ---------------------------------------------------------------- paged step

def _paged_problem(seed, lens, qlens, hq=4, hkv=2, d=8, bs=4, extra=3):
    rng = np.random.default_rng(seed)
    need = [(L + bs - 1) // bs for L in lens]
    nb = sum(need) + extra
    order = rng.permutation(nb).astype(np.int32)
    width = max(need)
    tables = np.full((len(lens), width), -1, np.int32)
    c = 0
    for b, n in enumerate(need):
        tables[b, :n] = order[c:c + n]
        c += n
    kc = rng.standard_normal((nb, bs, hkv, d))
    vc = rng.standard_normal((nb, bs, hkv, d))
    T = sum(qlens)
    q = rng.standard_normal((T, hq, d))
    qsl = np.concatenate([[0], np.cumsum(qlens)])
    return q, kc, vc, tables, qsl, np.array(lens)


def test_paged_step_matches_contiguous_attention_per_request():
    lens, qlens = [7, 13, 1, 9], [3, 1, 1, 9]
    q, kc, vc, tables, qsl, L = _paged_problem(30, lens, qlens)
    out, err, valid = oracle.paged_mixed_step(q, kc, vc, tables, qsl, L, 0.4)
    assert err == set() and valid.all()
    bs = kc.shape[1]
    for b in range(len(lens)):
        # contiguous K/V built by direct block reads, independent of gather()
        ids = tables[b, : (lens[b] + bs - 1) // bs]
        K = np.concatenate([kc[i] for i in ids])[: lens[b]]
        V = np.concatenate([vc[i] for i in ids])[: lens[b]]
        ref = _sdpa_reference(q[qsl[b]:qsl[b + 1]], K, V, 0.4, lens[b] - qlens[b])
        assert np.max(np.abs(out[qsl[b]:qsl[b + 1]] - ref)) < 1e-12


def test_paged_step_invariant_under_physical_block_permutation():
    lens, qlens = [11, 6, 17], [2, 1, 5]
    q, kc, vc, tables, qsl, L = _paged_problem(31, lens, qlens)
    out1, _, _ = oracle.paged_mixed_step(q, kc, vc, tables, qsl, L, 0.3)
    perm = np.random.default_rng(32).permutation(kc.shape[0])      # new id of old block i
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    tables2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1).astype(np.int32)
    out2, _, _ = oracle.paged_mixed_step(q, kc2, vc2, tables2, qsl, L, 0.3)
    assert np.array_equal(out1, out2)


def test_paged_decode_edge_cases():
    lens = [5, 0, 3]
    q, kc, vc, tables, qsl, L = _paged_problem(33, [5, 1, 3], [1, 1, 1])
    out, err, valid = oracle.paged_decode(q, kc, vc, tables, np.array(lens), 0.5)
    assert err == set() and valid.all()
    assert np.all(out[1] == 0)
    # a block id outside the pool is reported and leaves the row undefined
    bad = tables.copy()
    bad[2, 0] = kc.shape[0]
    out, err, valid = oracle.paged_decode(q, kc, vc, bad, np.array(lens), 0.5)
    assert err == {oracle.ERR_BLOCK_OOB} and not valid[2] and valid[0]
    # seq_len larger than the table
    out, err, valid = oracle.paged_decode(q, kc, vc, tables, np.array([5, 0, 99]), 0.5)
    assert err == {oracle.ERR_SEQ_TOO_LONG} and not valid[2]


def test_query_longer_than_sequence_is_an_error():
    q, kc, vc, tables, qsl, L = _paged_problem(34, [4, 4], [1, 1])
    out, err, valid = oracle.paged_mixed_step(q[:2], kc, vc, tables, [0, 2, 2], [1, 0], 0.5)
    assert err == {oracle.ERR_QUERY_TOO_LONG} and not valid.any()


def test_bf16_inputs_upcast_exactly():
    x = torch.randn(1000).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().astype(np.uint16)
    manual = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(x.to(torch.float64).numpy(), manual)


# ---------------------------------------------------------------- planted mistakes

def _pins_pass(mod):
    """Run a handful of the pins above against a (possibly mutated) oracle module."""
    q, K, V = _rand((5, 6, 8), 40), _rand((37, 3, 8), 41), _rand((37, 3, 8), 42)
    ok = np.max(np.abs(mod.attend_two_pass(q, K, V, 0.35, 32)
                       - _sdpa_reference(q, K, V, 0.35, 32))) < 1e-12
    ok &= np.max(np.abs(mod.attend_online(q, K, V, 0.35, 32, 5)
                        - _sdpa_reference(q, K, V, 0.35, 32))) < 1e-12
    ok &= np.max(np.abs(mod.attend_split(q, K, V, 0.35, 32, 3)
                        - _sdpa_reference(q, K, V, 0.35, 32))) < 1e-12
    g = _golden("slot_worked_example.json")
    ok &= mod.slot_of(g["block_table"], g["position"], g["block_size"]) == g["slot"]
    return bool(ok)


def test_pins_pass_on_the_real_oracle():
    assert _pins_pass(oatt)


@pytest.mark.parametrize("mutation", ["gqa_modulo", "causal_off_by_one", "no_rescale",
                                      "slot_uses_logical", "merge_without_weights",
                                      "scale_after_softmax"])
def test_pins_catch_planted_mistakes(mutation, monkeypatch):
    import importlib
    mod = importlib.reload(oatt)
    try:
        if mutation == "gqa_modulo":
            monkeypatch.setattr(mod, "_kv_head", lambda h, hq, hkv: h % hkv)
        elif mutation == "causal_off_by_one":
            orig = mod._scores
            monkeypatch.setattr(mod, "_scores", lambda q, k, s, fp: orig(q, k, s, fp - 1))
        elif mutation == "no_rescale":
            real_exp = np.exp

            def attend_online(q, K, V, scale, first_pos, tile=16):
                # forgets exp(m_old - m_new) on the running sums
                q, K, V = (np.asarray(a, dtype=np.float64) for a in (q, K, V))
                n_q, hq, d = q.shape
                out = np.zeros((n_q, hq, d))
                for h in range(hq):
                    kv = mod._kv_head(h, hq, K.shape[1])
                    s_all = mod._scores(q[:, h], K[:, kv], scale, first_pos)
                    m = np.full(n_q, -np.inf)
                    l = np.zeros(n_q)
                    o = np.zeros((n_q, d))
                    for j0 in range(0, K.shape[0], tile):
                        s = s_all[:, j0:j0 + tile]
                        m = np.maximum(m, s.max(axis=1))
                        p = real_exp(s - m[:, None])
                        l = l + p.sum(axis=1)
                        o = o + p @ V[j0:j0 + tile, kv]
                    out[:, h] = o / l[:, None]
                return out
            monkeypatch.setattr(mod, "attend_online", attend_online)
        elif mutation == "slot_uses_logical":
            monkeypatch.setattr(mod, "slot_of", lambda row, p, bs: (p // bs) * bs + p % bs)
        elif mutation == "merge_without_weights":
            def merge(parts):
                return sum(p[2] for p in parts) / sum(p[1] for p in parts)[..., None]
            monkeypatch.setattr(mod, "merge_partials", merge)
        elif mutation == "scale_after_softmax":
            orig = mod._scores
            monkeypatch.setattr(mod, "_scores", lambda q, k, s, fp: orig(q, k, 1.0, fp))
        assert not _pins_pass(mod)
    finally:
        monkeypatch.undo()
        importlib.reload(oatt)

"""Property-based pins of the CPU oracle (no GPU): the identities the fixed
cases in test_oracle.py pin, over shapes, lengths, scales and value ranges
drawn by hypothesis.

  * the two-pass softmax attention equals torch's scaled_dot_product_attention
    in float64 with an explicit bottom-right causal mask (a library routine);
  * the online (streaming) softmax equals the two-pass form for any tile;
  * split-KV partials merged by log-sum-exp equal the unsplit attention for
    any number of partitions, empty partitions included;
  * slot mapping through any block table and block size round-trips to
    (table[p // bs], p % bs) and writes every slot of the pool once.
"""

import math

import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle

SETTINGS = settings(max_examples=60, deadline=None, derandomize=True)


@st.composite
def attention_case(draw):
    hkv = draw(st.sampled_from([1, 2, 4]))
    g = draw(st.sampled_from([1, 2, 4, 8]))
    d = draw(st.sampled_from([1, 3, 8, 16]))
    L = draw(st.integers(1, 40))
    n_q = draw(st.integers(1, L))
    amp = draw(st.sampled_from([0.1, 1.0, 8.0]))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    q = amp * rng.standard_normal((n_q, hkv * g, d))
    K = amp * rng.standard_normal((L, hkv, d))
    V = rng.standard_normal((L, hkv, d))
    scale = draw(st.sampled_from([1 / math.sqrt(d), 0.05, 1.0]))
    return q, K, V, scale, L - n_q


def _sdpa(q, K, V, scale, first_pos):
    n_q, hq, d = q.shape
    L, hkv, _ = K.shape
    g = hq // hkv
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(g, 0)[None]
    vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(g, 0)[None]
    mask = torch.arange(L)[None, :] <= (first_pos + torch.arange(n_q))[:, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


@SETTINGS
@given(attention_case())
def test_two_pass_equals_library_sdpa(case):
    q, K, V, scale, first = case
    got = oracle.attend_two_pass(q, K, V, scale, first)
    assert np.max(np.abs(got - _sdpa(q, K, V, scale, first))) < 1e-10


@SETTINGS
@given(attention_case(), st.integers(1, 17))
def test_online_equals_two_pass(case, tile):
    q, K, V, scale, first = case
    a = oracle.attend_two_pass(q, K, V, scale, first)
    b = oracle.attend_online(q, K, V, scale, first, tile=tile)
    assert np.max(np.abs(a - b)) < 1e-10


@SETTINGS
@given(attention_case(), st.integers(1, 12))
def test_split_merge_equals_unsplit(case, parts):
    # more partitions than keys leaves some empty: their weight must be zero
    q, K, V, scale, first = case
    a = oracle.attend_two_pass(q, K, V, scale, first)
    b = oracle.attend_split(q, K, V, scale, first, parts)
    assert np.max(np.abs(a - b)) < 1e-10


@SETTINGS
@given(st.sampled_from([1, 2, 8, 16, 32]), st.integers(1, 12), st.integers(0, 2 ** 31 - 1))
def test_slot_mapping_round_trip(bs, nb, seed):
    order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    L = nb * bs
    slots = oracle.slot_mapping(order[None, :], [0, L], [L], bs)
    assert sorted(slots.tolist()) == list(range(L))
    for p, s in enumerate(slots.tolist()):
        assert (s // bs, s % bs) == (order[p // bs], p % bs)

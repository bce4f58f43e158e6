"""Pins of the block-management oracle (oracle/blocks.py): the slot build
against the pages' worked example and a brute-force walk of the pool, and
block copies through a copy-on-write fork that the attention oracle must see
consistently."""

import json
import os

import numpy as np
import pytest

import oracle
from oracle import blocks as BL

GOLD = os.path.join(os.path.dirname(__file__), "golden", "slot_worked_example.json")


def test_slot_build_worked_example():
    g = json.load(open(GOLD))
    table = np.array([g["block_table"]], dtype=np.int32)
    slots, err = BL.slot_mapping_positions(table, [0], [g["position"]], g["block_size"], 64)
    assert err == set() and int(slots[0]) == g["slot"]


def test_slot_build_brute_force_walk():
    """Every position of every request lands on the pool cell found by
    scanning the physical blocks in table order."""
    rng = np.random.default_rng(3)
    bs, nb = 8, 40
    perm = rng.permutation(nb)
    tables = np.stack([perm[:10], perm[10:20], perm[20:30]]).astype(np.int32)
    req = np.repeat(np.arange(3), 80)
    pos = np.tile(np.arange(80), 3)
    slots, err = BL.slot_mapping_positions(tables, req, pos, bs, nb)
    assert err == set()
    cells = {}
    for b in range(3):
        k = 0
        for blk in tables[b]:
            for off in range(bs):
                cells[(b, k)] = int(blk) * bs + off
                k += 1
    assert all(int(s) == cells[(int(b), int(p))] for s, b, p in zip(slots, req, pos))
    assert len(set(slots.tolist())) == len(slots)        # distinct cells


def test_slot_build_padding_and_errors():
    tables = np.array([[3, 1], [0, -1]], dtype=np.int32)
    slots, err = BL.slot_mapping_positions(tables, [-1, 0, 1, 1, 0, 2], [5, 17, 3, 20, 32, 0], 16, 4)
    assert slots.tolist() == [-1, 17, 3, -1, -1, -1]
    assert err == {oracle.ERR_BLOCK_OOB, BL.ERR_POS_OOB_TABLE}


def test_copy_blocks_bit_exact_and_untouched():
    rng = np.random.default_rng(4)
    kp = rng.standard_normal((6, 4, 2, 8)).astype(np.float32)
    vp = rng.standard_normal((6, 4, 2, 8)).astype(np.float32)
    k2, v2, err = BL.copy_blocks(kp, vp, [[1, 4], [2, 5], [0, 9]])
    assert err == {oracle.ERR_BLOCK_OOB}
    assert k2[4].tobytes() == kp[1].tobytes() and v2[5].tobytes() == vp[2].tobytes()
    for b in (0, 1, 2, 3):
        assert k2[b].tobytes() == kp[b].tobytes() and v2[b].tobytes() == vp[b].tobytes()


def test_copy_on_write_fork():
    """Request A forks into A and B (same table, shared blocks).  B appends a
    token into the shared, partly filled last block: copy that block to a free
    one, point B's table at the copy, then write.  A's attention is unchanged,
    B's sees its new token, and both agree on the shared history."""
    rng = np.random.default_rng(5)
    bs, nb, hkv, d, hq = 4, 8, 1, 8, 2
    kp = rng.standard_normal((nb, bs, hkv, d))
    vp = rng.standard_normal((nb, bs, hkv, d))
    table_a = np.array([6, 2], dtype=np.int32)            # 6 tokens: block 2 holds 2
    L = 6
    q = rng.standard_normal((1, hq, d))
    before, _, _ = oracle.paged_decode(q, kp, vp, table_a[None], np.array([L]), 0.5)
    table_b = table_a.copy()
    kp2, vp2, err = BL.copy_blocks(kp, vp, [[2, 5]])       # copy-on-write of the last block
    table_b[1] = 5
    k_new, v_new = rng.standard_normal((1, hkv, d)), rng.standard_normal((1, hkv, d))
    slot = oracle.slot_of(table_b, L, bs)                  # B's token at position 6
    kp3, vp3, _ = oracle.cache_write(kp2, vp2, k_new, v_new, np.array([slot]))
    after_a, _, _ = oracle.paged_decode(q, kp3, vp3, table_a[None], np.array([L]), 0.5)
    assert err == set() and np.array_equal(after_a, before)
    ka = oracle.gather(kp3, table_a, L)
    kb = oracle.gather(kp3, table_b, L + 1)
    assert np.array_equal(kb[:L], ka) and np.array_equal(kb[L], k_new[0])
    # without the copy, the write would have changed A's block
    kp4, _, _ = oracle.cache_write(kp, vp, k_new, v_new, np.array([oracle.slot_of(table_a, L, bs)]))
    assert not np.array_equal(kp4[2], kp[2])


@pytest.mark.parametrize("mutation", ["offset_dropped", "copy_one_pool"])
def test_pins_catch_planted_mistakes(mutation, monkeypatch):
    good_copy = BL.copy_blocks
    if mutation == "offset_dropped":
        monkeypatch.setattr(BL, "slot_of", lambda row, p, bs: int(row[p // bs]) * bs)
    else:
        def bad(k_pool, v_pool, mapping):
            kp, vp, e = good_copy(k_pool, v_pool, mapping)
            return kp, np.array(v_pool, copy=True), e
        monkeypatch.setattr(BL, "copy_blocks", bad)
    failed = 0
    for fn in (test_slot_build_worked_example, test_slot_build_brute_force_walk,
               test_copy_blocks_bit_exact_and_untouched):
        try:
            fn()
        except AssertionError:
            failed += 1
    monkeypatch.undo()
    assert failed > 0, mutation

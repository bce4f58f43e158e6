"""Pins of the rotary-embedding oracle (oracle/rope.py) against facts that do
not come from the oracle itself: the complex-plane form the pages describe
(evaluated with Python's cmath, one pair at a time), closed forms, the
relative-position identity, norm preservation, and planted mistakes."""

import cmath
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import rope as R

GOLD = os.path.join(os.path.dirname(__file__), "golden", "llama3_8b_rope.json")


def _x(T, H, D, seed=0):
    return np.random.default_rng(seed).standard_normal((T, H, D))


@pytest.mark.parametrize("neox", [True, False])
@pytest.mark.parametrize("rot", [8, 16])
def test_complex_plane_form(neox, rot):
    """Each pair (x1, x2) as x1 + i x2, multiplied by e^{i p theta_i}."""
    D, theta = 16, 10000.0
    x = _x(5, 2, D, 1)
    pos = np.array([0, 1, 7, 100, 4095])
    table = R.cos_sin_table(4096, rot, theta)
    got = R.rotate(x, pos, table, rot, neox)
    half = rot // 2
    for t in range(5):
        for h in range(2):
            want = list(x[t, h])
            for i in range(half):
                a, b = (i, i + half) if neox else (2 * i, 2 * i + 1)
                ang = int(pos[t]) * theta ** (-2.0 * i / rot)
                z = complex(x[t, h, a], x[t, h, b]) * cmath.exp(1j * ang)
                want[a], want[b] = z.real, z.imag
            assert np.allclose(got[t, h], want, rtol=0, atol=1e-12)


def test_position_zero_is_identity():
    x = _x(3, 4, 32)
    table = R.cos_sin_table(8, 32, 500000.0)
    for neox in (True, False):
        assert np.array_equal(R.rotate(x, [0, 0, 0], table, 32, neox), x)


def test_first_pair_turns_by_one_radian_per_position():
    """Pair 0 has frequency theta**0 = 1: position p turns e1 to (cos p, sin p)."""
    D = 8
    x = np.zeros((1, 1, D))
    x[0, 0, 0] = 1.0
    table = R.cos_sin_table(10, D, 10000.0)
    for p in range(10):
        y = R.rotate(x, [p], table, D, neox=False)
        assert abs(y[0, 0, 0] - math.cos(p)) < 1e-15 and abs(y[0, 0, 1] - math.sin(p)) < 1e-15
        yn = R.rotate(x, [p], table, D, neox=True)
        assert abs(yn[0, 0, 0] - math.cos(p)) < 1e-15 and abs(yn[0, 0, D // 2] - math.sin(p)) < 1e-15


def test_frequencies_geometric_from_theta():
    g = json.load(open(GOLD))
    f = R.inv_freq(g["rotary_dim"], g["rope_theta"])
    assert f[0] == 1.0 and len(f) == g["rotary_dim"] // 2
    ratio = g["rope_theta"] ** (-2.0 / g["rotary_dim"])
    assert np.allclose(f[1:] / f[:-1], ratio, rtol=1e-13, atol=0)
    assert abs(f[-1] - g["rope_theta"] ** (-(g["rotary_dim"] - 2) / g["rotary_dim"])) < 1e-18


def test_table_is_angle_additive():
    """row(p + q) from rows p and q by the addition formulas."""
    t = R.cos_sin_table(64, 16, 500000.0)
    h = 8
    for p, q in [(3, 5), (10, 50), (31, 32)]:
        c = t[p, :h] * t[q, :h] - t[p, h:] * t[q, h:]
        s = t[p, h:] * t[q, :h] + t[p, :h] * t[q, h:]
        assert np.allclose(c, t[p + q, :h], atol=1e-14) and np.allclose(s, t[p + q, h:], atol=1e-14)


@pytest.mark.parametrize("neox", [True, False])
def test_relative_position_identity(neox):
    """<R_m q, R_n k> depends on m - n only (the pages' point about RoPE)."""
    D = 64
    q, k = _x(1, 1, D, 2), _x(1, 1, D, 3)
    table = R.cos_sin_table(5000, D, 500000.0)
    for m, n, s in [(10, 3, 100), (0, 7, 4000), (1234, 1234, 17)]:
        a = float(np.dot(R.rotate(q, [m], table, D, neox)[0, 0], R.rotate(k, [n], table, D, neox)[0, 0]))
        b = float(np.dot(R.rotate(q, [m + s], table, D, neox)[0, 0],
                         R.rotate(k, [n + s], table, D, neox)[0, 0]))
        assert abs(a - b) < 1e-10


def test_norm_preserved_and_partial_rotary():
    x = _x(6, 3, 128, 4)
    table = R.cos_sin_table(1 << 15, 64, 500000.0)
    pos = [5, 77, 1000, 20000, 32767, 1]
    for neox in (True, False):
        y = R.rotate(x, pos, table, 64, neox)
        assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), atol=1e-12)
        assert np.array_equal(y[..., 64:], x[..., 64:])


def test_split_half_equals_adjacent_after_permutation():
    """neox pairs (i, i + d/2) are the adjacent pairs of the interleaved view."""
    D = 32
    x = _x(4, 2, D, 5)
    perm = np.empty(D, dtype=int)
    perm[0::2] = np.arange(D // 2)
    perm[1::2] = np.arange(D // 2) + D // 2
    table = R.cos_sin_table(100, D, 10000.0)
    pos = [0, 9, 50, 99]
    a = R.rotate(x, pos, table, D, True)
    b = R.rotate(x[..., perm], pos, table, D, False)
    assert np.allclose(a[..., perm], b, atol=1e-14)


def test_cache_write_places_rotated_k_and_plain_v():
    T, Hq, Hkv, D, nb, bs = 7, 4, 2, 16, 4, 4
    rng = np.random.default_rng(6)
    q, k, v = rng.standard_normal((T, Hq, D)), rng.standard_normal((T, Hkv, D)), rng.standard_normal((T, Hkv, D))
    kp, vp = rng.standard_normal((nb, bs, Hkv, D)), rng.standard_normal((nb, bs, Hkv, D))
    pos = np.array([0, 3, 9, 15, 40, 2, 8])
    slots = np.array([5, -1, 0, 15, 7, 99, 3])     # -1 padding, 99 past the pool
    table = R.cos_sin_table(16, D, 10000.0)        # position 40 is past the table
    qr, kp2, vp2, err, ok = R.rope_cache_write(q, k, v, pos, slots, kp, vp, table, D, True)
    assert err == {R.ERR_POS_OOB, "slot_out_of_range"}
    assert list(ok) == [True, True, True, True, False, True, True]
    assert np.array_equal(qr[4], q[4])                                   # not rotated
    assert np.array_equal(vp2[1, 1], v[0]) and np.array_equal(vp2[3, 3], v[3])
    assert np.array_equal(vp2[1, 3], vp[1, 3])                           # slot 7: token 4 skipped
    assert np.allclose(kp2[0, 3], R.rotate(k[6:7], [8], table, D, True)[0], atol=0)
    untouched = np.ones((nb, bs), bool)
    for s in (5, 0, 15, 3):
        untouched[s // bs, s % bs] = False
    assert np.array_equal(kp2[untouched], kp[untouched])


# ---------------------------------------------------------------- planted mistakes

@pytest.mark.parametrize("mutation", ["sine_sign", "halves_swapped", "freq_exponent", "pairing"])
def test_pins_catch_planted_mistakes(mutation, monkeypatch):
    good_table, good_rot, good_pairs = R.cos_sin_table, R.rotate, R.pair_index
    if mutation == "sine_sign":
        def rot(x, positions, table, rotary_dim, neox):
            t2 = table.copy()
            t2[:, rotary_dim // 2:rotary_dim] *= -1
            return good_rot(x, positions, t2, rotary_dim, neox)
        monkeypatch.setattr(R, "rotate", rot)
    elif mutation == "halves_swapped":
        monkeypatch.setattr(R, "cos_sin_table", lambda m, r, th: np.roll(good_table(m, r, th), r // 2, axis=1))
    elif mutation == "freq_exponent":
        monkeypatch.setattr(R, "inv_freq",
                            lambda r, th: np.power(np.float64(th), -np.arange(r // 2) / r))
    elif mutation == "pairing":
        monkeypatch.setattr(R, "pair_index", lambda r, neox: good_pairs(r, not neox))
    failed = 0
    for fn, args in [(test_complex_plane_form, (True, 16)), (test_complex_plane_form, (False, 8)),
                     (test_first_pair_turns_by_one_radian_per_position, ()),
                     (test_frequencies_geometric_from_theta, ())]:
        try:
            fn(*args)
        except AssertionError:
            failed += 1
    monkeypatch.undo()
    assert failed > 0, mutation

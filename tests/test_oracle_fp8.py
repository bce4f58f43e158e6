"""Pins of the e4m3 oracle (oracle/fp8.py): the decode table and the
rounding against torch's float8_e4m3fn conversion (a library routine),
hand-checked ties and saturation, the error bound of 3 mantissa bits, and a
pool whose values are on the e4m3 grid giving the unquantised attention."""

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8 as F


def test_decode_table_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = F.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2      # 0x7F, 0xFF
    assert np.array_equal(ours[~nan], lib[~nan])
    assert np.nanmax(ours) == 448.0 and ours[1] == 2.0 ** -9 and ours[8] == 2.0 ** -6


def test_encode_matches_torch_in_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 40,
        rng.uniform(-2.0 ** -5, 2.0 ** -5, 50000).astype(np.float32),     # subnormal range
        (F.e4m3_decode(np.arange(256, dtype=np.uint8)[:126]) +
         np.diff(F.e4m3_decode(np.arange(127, dtype=np.uint8))) / 2).astype(np.float32),  # midpoints
    ])
    x = x[np.abs(x) <= 448]
    ours = F.e4m3_encode(x.astype(np.float64))
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # torch keeps the sign of values that round to zero; so do we
    assert np.array_equal(ours, lib)


def test_ties_to_even_and_saturation():
    enc = lambda v: int(F.e4m3_encode(np.array([v]))[0])
    assert enc(1.0625) == 0x38 and enc(1.1875) == 0x3A          # 1 + 1/16 -> 1, 1 + 3/16 -> 1.25
    assert enc(2.0 ** -10) == 0x00 and enc(3 * 2.0 ** -10) == 0x02
    assert enc(464.0) == 0x7E and enc(1e9) == 0x7E and enc(-1e9) == 0xFE
    assert enc(-0.0) == 0x80 and enc(0.0) == 0x00


def test_quantisation_error_bound():
    rng = np.random.default_rng(8)
    scale = 0.0171
    x = rng.standard_normal(100000).astype(np.float32)
    back = F.dequantize(F.quantize(x, scale), scale)
    s32 = float(np.float32(scale))
    assert np.all(np.abs(back - x) <= 2.0 ** -4 * np.abs(x) + 2.0 ** -10 * s32 + 1e-12)


def test_grid_values_attend_exactly():
    """Pools whose values are e4m3 codes times the scale: the fp8 pool and
    its float64 dequantisation give the same attention as the values
    themselves."""
    rng = np.random.default_rng(9)
    nb, bs, hkv, d, scale = 6, 4, 2, 8, 0.25
    codes = rng.integers(0, 126, (nb, bs, hkv, d)).astype(np.uint8) | \
        (rng.integers(0, 2, (nb, bs, hkv, d)).astype(np.uint8) << 7)
    vals = F.e4m3_decode(codes) * scale
    assert np.array_equal(F.quantize(vals.astype(np.float32), scale), np.where(vals == 0, codes & 0x80, codes))
    q = rng.standard_normal((2, 4, d))
    tables = np.array([[0, 1, 2], [3, 4, 5]], dtype=np.int32)
    lens = np.array([10, 12])
    a, _, _ = oracle.paged_decode(q, vals, vals, tables, lens, 0.3)
    b, _, _ = oracle.paged_decode(q, F.dequantize(codes, scale), F.dequantize(codes, scale),
                                  tables, lens, 0.3)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("mutation", ["bias", "no_even_ties", "no_saturation"])
def test_pins_catch_planted_mistakes(mutation, monkeypatch):
    good_dec, good_enc = F.e4m3_decode, F.e4m3_encode
    if mutation == "bias":
        monkeypatch.setattr(F, "e4m3_decode", lambda c: good_dec(c) * 2.0)
    elif mutation == "no_even_ties":
        def enc(x):
            x = np.asarray(x, dtype=np.float64)
            return good_enc(np.nextafter(x, np.sign(x) * np.inf))     # ties away from zero
        monkeypatch.setattr(F, "e4m3_encode", enc)
    else:
        monkeypatch.setattr(F, "e4m3_encode",
                            lambda x: np.where(np.abs(np.asarray(x)) > 448, np.uint8(0x7F),
                                               good_enc(np.clip(x, -448, 448))).astype(np.uint8))
    failed = 0
    for fn in (test_decode_table_matches_torch, test_encode_matches_torch_in_range,
               test_ties_to_even_and_saturation):
        try:
            fn()
        except AssertionError:
            failed += 1
    monkeypatch.undo()
    assert failed > 0, mutation

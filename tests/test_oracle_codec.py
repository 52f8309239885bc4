"""Pins for the oracle's 4-bit group codec, checked against things other than itself.

The codec follows the flashloop 0.1.0 PyPI description ("Configuration and
supported scope": 4-bit K/V, group size 64) and the flozi guide "FlashLoop:
store changes between repeated passes", section 3 (group-wise asymmetric,
per-channel keys, per-token values).
"""
import struct
from fractions import Fraction

import numpy as np
import pytest

from oracle import flashloop_oracle as fo


def _half_struct(x: float) -> np.float16:
    """binary16 rounding done by CPython's own packer (independent of NumPy)."""
    return np.frombuffer(struct.pack("<e", x), dtype=np.float16)[0]


def test_half_rn_matches_cpython_packer():
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 3,
        rng.standard_normal(1000).astype(np.float32) * 1e-5,      # binary16 subnormals
        np.float32([1 + 2 ** -11, 1 + 3 * 2 ** -11, 2049.0, 2051.0, 6.1e-5, 0.0, -0.0]),  # ties
    ])
    mine = fo.half_rn(vals)
    ref = np.array([_half_struct(float(v)) for v in vals], dtype=np.float16)
    assert np.array_equal(mine.view(np.uint16), ref.view(np.uint16))


def test_hand_example_half_steps():
    x = np.tile(np.arange(16, dtype=np.float32) * 0.5, 4)
    codes, s, z = fo.quantize(x)
    assert float(s) == 0.5 and float(z) == 0.0
    assert np.array_equal(codes, np.tile(np.arange(16), 4))
    assert np.array_equal(fo.dequant(codes, s, z), x)


def test_constant_group_has_zero_scale():
    x = np.full(64, 0.3, np.float32)
    codes, s, z = fo.quantize(x)
    assert float(s) == 0.0 and not codes.any()
    assert np.all(fo.dequant(codes, s, z) == np.float32(_half_struct(0.3)))


def _levels(s, z):
    return np.float64(z) + np.arange(16, dtype=np.float64) * np.float64(s)


@pytest.mark.parametrize("scale", [1.0, 0.05, 30.0])
def test_codes_are_nearest_levels_by_brute_force(scale):
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((200, 64)) * scale).astype(np.float32)
    codes, s, z = fo.quantize(x, axis=1)
    for g in range(x.shape[0]):
        lv = _levels(s[g], z[g])
        dist = np.abs(x[g].astype(np.float64)[:, None] - lv[None, :])
        best = dist.min(axis=1)
        chosen = dist[np.arange(64), codes[g]]
        assert np.all(chosen <= best + 1e-6 * float(s[g]))


def test_scale_and_zero_against_exact_arithmetic():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((300, 64)).astype(np.float32)
    _, s, z = fo.quantize(x, axis=1)
    for g in range(x.shape[0]):
        mn, mx = float(x[g].min()), float(x[g].max())
        assert z[g].view(np.uint16) == _half_struct(mn).view(np.uint16)
        exact = (Fraction(mx) - Fraction(mn)) / 15
        ulp = np.spacing(np.float16(s[g]))
        assert abs(Fraction(float(s[g])) - exact) <= Fraction(float(ulp)) * Fraction(1, 2) * (1 + Fraction(1, 8192))


def test_min_and_max_take_end_codes():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((500, 64)).astype(np.float32)
    codes, _, _ = fo.quantize(x, axis=1)
    rows = np.arange(500)
    assert np.all(codes[rows, x.argmin(axis=1)] == 0)
    assert np.all(codes[rows, x.argmax(axis=1)] == 15)


def test_reconstruction_maps_back_to_its_own_code():
    rng = np.random.default_rng(14)
    x = rng.standard_normal((100, 64)).astype(np.float32)
    codes, s, z = fo.quantize(x, axis=1)
    xh = fo.dequant(codes, s[:, None], z[:, None])
    for g in range(100):
        lv = _levels(s[g], z[g])
        near = np.abs(xh[g].astype(np.float64)[:, None] - lv[None, :]).argmin(axis=1)
        assert np.array_equal(near, codes[g])


def _correctly_rounded_f32(v: Fraction) -> np.float32:
    c = np.float32(float(v))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    errs = [abs(Fraction(float(t)) - v) for t in cands]
    best = min(errs)
    ties = [t for t, e in zip(cands, errs) if e == best]
    if len(ties) == 1:
        return ties[0]
    return [t for t in ties if (t.view(np.uint32) & 1) == 0][0]


def test_dequant_is_one_rounding_of_the_exact_value():
    rng = np.random.default_rng(15)
    s = fo.half_rn(rng.uniform(1e-3, 2.0, 400))
    z = fo.half_rn(rng.standard_normal(400) * 3)
    c = rng.integers(0, 16, 400).astype(np.uint8)
    got = fo.dequant(c, s, z)
    for i in range(400):
        exact = Fraction(int(c[i])) * Fraction(float(s[i])) + Fraction(float(z[i]))
        assert got[i] == _correctly_rounded_f32(exact)


def test_base_groups_keys_per_channel_and_values_per_token_half():
    H, T, D = 2, 128, 128
    t = np.arange(T)[None, :, None]
    c = np.arange(D)[None, None, :]
    K = np.broadcast_to(0.5 * (t % 16) + 2.0 * (c % 64), (H, T, D)).astype(np.float32)
    V = np.broadcast_to(0.25 * (c % 16) + 0.125 * (t % 64), (H, T, D)).astype(np.float32)
    enc = fo.encode_base(K, V)
    assert np.all(enc["ks"].astype(np.float32) == 0.5)
    assert np.array_equal(enc["kz"][0, 0].astype(np.float32), 2.0 * (np.arange(D) % 64))
    assert np.array_equal(enc["kc"][0, :, 5], np.arange(T) % 16)
    assert np.all(enc["vs"].astype(np.float32) == 0.25)
    assert np.array_equal(enc["vz"][1, :, 1].astype(np.float32), 0.125 * (np.arange(T) % 64))
    assert np.array_equal(enc["vc"][1, 3], np.arange(D) % 16)
    kh, vh = fo.decode_base(enc)
    assert np.array_equal(kh, K) and np.array_equal(vh, V)


def test_residual_key_groups_are_64_consecutive_slots_with_partial_tail():
    H, n, D = 1, 100, 128
    i = np.arange(n, dtype=np.float32)[None, :, None]
    EK = np.broadcast_to(0.25 * i, (H, n, D)).astype(np.float32)
    EV = np.zeros((H, n, D), np.float32)
    enc = fo.encode_residual(EK, EV)
    assert enc["ks"].shape == (1, 2, D)
    assert float(enc["kz"][0, 0, 0]) == 0.0
    assert float(enc["kz"][0, 1, 0]) == 16.0          # min over slots 64..99 only
    assert float(enc["ks"][0, 1, 0]) == float(fo.half_rn(np.float32(8.75) / np.float32(15)))
    assert not enc["vc"].any() and not enc["vs"].astype(np.float32).any()

"""Pins for the oracle's codec variants of the loop r >= 2 stores.

Sources: flozi guide "FlashLoop: store changes between repeated passes", section 4
(the "Per-loop KIVI4" ablation row quantises full KV states directly instead of the
cross-loop residuals; the 2-bit row of Figure 5) and section 2 (residuals between
adjacent loops shrink, so quantising them loses less than quantising the full state
at the same bit budget); FlashLoop project page, "Experiments", caption of Figure 5
(residual quantisation precision varied, other components fixed).

Each pin is fixed by arithmetic done here independently: hand-made groups on exact
grids, brute force over the four 2-bit levels, exact rational arithmetic for the
scale, a store that must equal the (separately pinned) base encoder, and the pages'
error ordering.  A 2-bit quantiser with the wrong level count, a full-state store that
still subtracts the previous loop, or one whose reconstruction keeps adding earlier
stores fails one of them.
"""
from fractions import Fraction
import struct

import numpy as np
import pytest

from oracle import flashloop_oracle as fo


def _half(x: float) -> np.float16:
    return np.frombuffer(struct.pack("<e", x), dtype=np.float16)[0]


# ---- the 2-bit quantiser ------------------------------------------------------
def test_int2_hand_example():
    x = np.tile(np.float32([0.0, 0.5, 1.0, 1.5]), 16)
    codes, s, z = fo.quantize(x, levels=fo.LEVELS2)
    assert float(s) == 0.5 and float(z) == 0.0
    assert np.array_equal(codes, np.tile(np.arange(4), 16))
    assert np.array_equal(fo.dequant(codes, s, z), x)


@pytest.mark.parametrize("scale", [1.0, 0.02, 40.0])
def test_int2_codes_are_nearest_of_four_levels(scale):
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((200, 64)) * scale).astype(np.float32)
    codes, s, z = fo.quantize(x, axis=1, levels=fo.LEVELS2)
    assert codes.max() <= 3
    for g in range(x.shape[0]):
        lv = np.float64(z[g]) + np.arange(4, dtype=np.float64) * np.float64(s[g])
        dist = np.abs(x[g].astype(np.float64)[:, None] - lv[None, :])
        chosen = dist[np.arange(64), codes[g]]
        assert np.all(chosen <= dist.min(axis=1) + 1e-6 * float(s[g]))


def test_int2_scale_is_a_third_of_the_range_rounded_once():
    rng = np.random.default_rng(22)
    x = rng.standard_normal((300, 64)).astype(np.float32)
    codes, s, z = fo.quantize(x, axis=1, levels=fo.LEVELS2)
    rows = np.arange(300)
    assert np.all(codes[rows, x.argmin(axis=1)] == 0) and np.all(codes[rows, x.argmax(axis=1)] == 3)
    for g in range(300):
        mn, mx = float(x[g].min()), float(x[g].max())
        assert z[g].view(np.uint16) == _half(mn).view(np.uint16)
        exact = (Fraction(mx) - Fraction(mn)) / 3
        ulp = np.spacing(np.float16(s[g]))
        assert abs(Fraction(float(s[g])) - exact) <= Fraction(float(ulp)) * Fraction(1, 2) * (1 + Fraction(1, 8192))


# ---- per-loop full-state (KIVI4) stores -----------------------------------------
def _states(rng, H, n, loops, drift):
    """Loop states that drift from loop to loop: X^(r) = X^(r-1) + drift * noise."""
    K = [None, (rng.standard_normal((H, n, 128)) * 2).astype(np.float32)]
    V = [None, rng.standard_normal((H, n, 128)).astype(np.float32)]
    for _ in range(2, loops + 1):
        K.append((K[-1] + drift * rng.standard_normal((H, n, 128))).astype(np.float32))
        V.append((V[-1] + drift * rng.standard_normal((H, n, 128))).astype(np.float32))
    return K, V


def _layer(codec, K, V, sets, n):
    H, R = K[1].shape[0], len(K) - 1
    lay = fo.OracleLayer(H, R, n + 64, codec=codec)
    lay.encode_base(0, K[1], V[1])
    for r in range(2, R + 1):
        rows = sets[r]
        lay.encode_residual(r, rows, K[r][:, rows], V[r][:, rows])
    return lay


def test_full_state_store_of_all_tokens_is_the_base_encoding_of_that_loop():
    rng = np.random.default_rng(23)
    H, n = 2, 192
    K, V = _states(rng, H, n, 3, 0.1)
    every = np.arange(n)
    lay = _layer(fo.FULL_INT4, K, V, [None, every, every, every], n)
    for r in (2, 3):
        enc = lay.calls[r][0]["enc"]
        ref = fo.encode_base(K[r], V[r])    # all tokens active: slots = tokens
        for key in ("kc", "vc", "ks", "kz", "vs", "vz"):
            assert np.array_equal(np.asarray(enc[key]).view(np.uint8), np.asarray(ref[key]).view(np.uint8)), (r, key)
        kh, vh = fo.decode_base(ref)
        assert np.array_equal(lay.khat[r][:, :n], kh) and np.array_equal(lay.vhat[r][:, :n], vh)


def test_full_state_reconstruction_is_the_last_store_alone():
    rng = np.random.default_rng(24)
    H, n = 1, 128
    K, V = _states(rng, H, n, 4, 0.2)
    sets = [None, np.arange(n), np.arange(0, n, 2), np.arange(0, n, 4), np.arange(0, n, 8)]
    lay = _layer(fo.FULL_INT4, K, V, sets, n)
    # other loop-2 states: the loop-3 and loop-4 stores (and their tokens) do not change
    K2 = [k.copy() if k is not None else None for k in K]
    K2[2] = K2[2] + 5.0
    lay2 = _layer(fo.FULL_INT4, K2, V, sets, n)
    for r in (3, 4):
        assert np.array_equal(lay.khat[r][:, sets[r]], lay2.khat[r][:, sets[r]])
    # a token of depth 2 keeps its loop-2 store in loops 3 and 4; depth 3 its loop-3 store
    enc2 = lay.calls[2][0]["enc"]
    kh2, _ = fo.decode_residual(enc2)
    d2 = np.setdiff1d(sets[2], sets[3])
    pos = np.searchsorted(sets[2], d2)
    assert np.array_equal(lay.khat[4][:, d2], kh2[:, pos])
    # and the base reconstruction for tokens never updated after loop 1
    d1 = np.setdiff1d(np.arange(n), sets[2])
    assert np.array_equal(lay.khat[4][:, d1], lay.khat[1][:, d1])


# ---- INT2 residual stores ------------------------------------------------------
def test_int2_residual_on_an_exact_grid_reconstructs_exactly():
    H, n = 1, 64
    t = np.arange(n, dtype=np.float32)[None, :, None]
    c = np.arange(128, dtype=np.float32)[None, None, :]
    K1 = np.broadcast_to((t % 16) + 0 * c, (H, n, 128)).astype(np.float32)      # 4-bit grid: exact base
    V1 = np.broadcast_to((c % 16) * 0.5 + 0 * t, (H, n, 128)).astype(np.float32)
    E = np.broadcast_to(0.25 * ((t + c) % 4), (H, n, 128)).astype(np.float32)     # 2-bit grid, s = 0.25
    lay = fo.OracleLayer(H, 2, n + 64, codec=fo.RESIDUAL_INT2)
    lay.encode_base(0, K1, V1)
    assert np.array_equal(lay.khat[1][:, :n], K1) and np.array_equal(lay.vhat[1][:, :n], V1)
    lay.encode_residual(2, np.arange(n), K1 + E, V1 + E)
    enc = lay.calls[2][0]["enc"]
    assert enc["kc"].max() == 3 and np.all(enc["ks"].astype(np.float32) == 0.25)
    assert np.array_equal(lay.khat[2][:, :n], K1 + E) and np.array_equal(lay.vhat[2][:, :n], V1 + E)
    # the 4-bit codec spreads the same range over 15 steps: scale fp16(0.75 / 15)
    lay4 = fo.OracleLayer(H, 2, n + 64)
    lay4.encode_base(0, K1, V1)
    lay4.encode_residual(2, np.arange(n), K1 + E, V1 + E)
    want = _half(float(np.float32(0.75) / np.float32(15))).view(np.uint16)
    assert np.all(lay4.calls[2][0]["enc"]["ks"].view(np.uint16) == want)


def test_int2_residual_error_is_within_half_a_step():
    rng = np.random.default_rng(25)
    H, n = 2, 256
    K, V = _states(rng, H, n, 2, 0.3)
    lay = _layer(fo.RESIDUAL_INT2, K, V, [None, np.arange(n), np.arange(n)], n)
    enc = lay.calls[2][0]["enc"]
    ks = enc["ks"].astype(np.float64)                       # [H][4][128]
    err = np.abs(lay.khat[2][:, :n].astype(np.float64) - K[2])
    step = np.repeat(ks, 64, axis=1)
    # half a step, plus the fp32 roundings of the residual, the fma and the add
    assert np.all(err <= 0.5 * step + 4e-6 * (1 + np.abs(K[2])))
    assert enc["kc"].max() == 3 and enc["vc"].max() == 3


def test_error_ordering_the_pages_report():
    """Residual INT4 beats full-state INT4 when the loops drift little (and more so with
    depth); INT2 residuals lose more than INT4 residuals."""
    rng = np.random.default_rng(26)
    H, n, R = 2, 256, 4
    K, V = _states(rng, H, n, R, 0.05)
    every = np.arange(n)
    sets = [None] + [every] * R
    err = {}
    for codec in (fo.RESIDUAL_INT4, fo.FULL_INT4, fo.RESIDUAL_INT2):
        lay = _layer(codec, K, V, sets, n)
        err[codec] = [float(np.sqrt(np.mean((lay.khat[r][:, :n] - K[r]) ** 2))) for r in range(1, R + 1)]
    for r in range(1, R):
        assert err[fo.RESIDUAL_INT4][r] < err[fo.FULL_INT4][r]
        assert err[fo.RESIDUAL_INT4][r] < err[fo.RESIDUAL_INT2][r]
    assert err[fo.RESIDUAL_INT4][0] == err[fo.FULL_INT4][0] == err[fo.RESIDUAL_INT2][0]   # same base

"""Pins for the oracle's sparse prefill attention (causal attention of the active
tokens of one loop over every token's key/value).

Sources: FlashLoop project page, "The Method", Step 01 (only the active tokens are
recomputed in a token-sparse loop) and the paragraph after Step 03 (selected tokens
gathered into compact buffers so the work stays a regular GEMM).
"""
import math

import numpy as np
import pytest
import torch

from oracle import flashloop_oracle as fo


def _brute(q, K, V, p):
    """One query row, Python floats and loops."""
    D = len(q)
    ls = [sum(float(q[d]) * float(K[j][d]) for d in range(D)) / math.sqrt(D) for j in range(p + 1)]
    m = max(ls)
    e = [math.exp(x - m) for x in ls]
    t = sum(e)
    return [sum(e[j] / t * float(V[j][d]) for j in range(p + 1)) for d in range(D)]


def test_brute_force_rows():
    rng = np.random.default_rng(3)
    H, N, D = 2, 9, 6
    K = rng.standard_normal((H, N, D))
    V = rng.standard_normal((H, N, D))
    pos = np.array([0, 3, 4, 8])
    q = rng.standard_normal((H, len(pos), D))
    o = fo.prefill_attention(q, pos, K, V)
    for h in range(H):
        for i, p in enumerate(pos):
            assert np.allclose(o[h, i], _brute(q[h, i], K[h], V[h], int(p)), rtol=1e-12, atol=1e-12)


def test_first_token_sees_only_itself():
    rng = np.random.default_rng(4)
    K = rng.standard_normal((1, 5, 8))
    V = rng.standard_normal((1, 5, 8))
    q = rng.standard_normal((1, 1, 8)) * 100.0
    assert np.array_equal(fo.prefill_attention(q, [0], K, V)[0, 0], V[0, 0])


def test_all_active_is_causal_attention():
    torch.manual_seed(5)
    H, N, D = 3, 37, 128
    q = torch.randn(H, N, D, dtype=torch.float64)
    K = torch.randn(H, N, D, dtype=torch.float64)
    V = torch.randn(H, N, D, dtype=torch.float64)
    ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, is_causal=True)
    o = fo.prefill_attention(q.numpy(), np.arange(N), K.numpy(), V.numpy())
    assert np.allclose(o, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_rows_are_independent_and_causal():
    rng = np.random.default_rng(6)
    H, N, D = 2, 30, 16
    K = rng.standard_normal((H, N, D))
    V = rng.standard_normal((H, N, D))
    pos = np.array([2, 7, 11, 20])
    q = rng.standard_normal((H, len(pos), D))
    o = fo.prefill_attention(q, pos, K, V)
    # one row alone gives the same answer as within the active set
    assert np.array_equal(fo.prefill_attention(q[:, 2:3], pos[2:3], K, V)[:, 0], o[:, 2])
    # keys after the last active position do not matter
    K2, V2 = K.copy(), V.copy()
    K2[:, 21:] = 1e3
    V2[:, 21:] = -1e3
    assert np.array_equal(fo.prefill_attention(q, pos, K2, V2), o)
    # a key inside a row's window does matter
    K2[:, 5] += 1.0
    assert not np.allclose(fo.prefill_attention(q, pos, K2, V)[:, 1], o[:, 1])

"""Pins for the oracle's encoders, attention and loop-aware sparse attention.

Sources: FlashLoop project page, "The Method", Step 02 (select columns from the
preceding loop, keep their global probability mass) and Step 03 (residual
relative to the reconstructed state of the preceding loop); flozi guide
"FlashLoop: store changes between repeated passes", section 3.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import flashloop_oracle as fo


def _brute_attention(q, K, V):
    """Textbook single-query softmax attention with Python floats and loops."""
    N, D = K.shape
    ls = [sum(float(q[d]) * float(K[j, d]) for d in range(D)) / math.sqrt(D) for j in range(N)]
    mx = max(ls)
    e = [math.exp(v - mx) for v in ls]
    tot = sum(e)
    p = [v / tot for v in e]
    o = [sum(p[j] * float(V[j, d]) for j in range(N)) for d in range(D)]
    return np.array(o), np.array(p)


@pytest.mark.parametrize("N", [1, 7, 40])
def test_dense_attention_matches_brute_force(N):
    rng = np.random.default_rng(N)
    H, D = 2, fo.HEAD_DIM
    q = rng.standard_normal((H, D)).astype(np.float32)
    K = rng.standard_normal((H, N, D)).astype(np.float32)
    V = rng.standard_normal((H, N, D)).astype(np.float32)
    o, p, _ = fo.attention_dense(q, K, V)
    for h in range(H):
        ob, pb = _brute_attention(q[h], K[h], V[h])
        assert np.allclose(p[h], pb, rtol=1e-12, atol=1e-15)
        assert np.allclose(o[h], ob, rtol=1e-11, atol=1e-13)


def test_equal_logits_give_uniform_weights():
    K = np.random.default_rng(1).standard_normal((1, 33, fo.HEAD_DIM)).astype(np.float32)
    _, p, _ = fo.attention_dense(np.zeros((1, fo.HEAD_DIM), np.float32), K, K)
    assert np.allclose(p, 1.0 / 33, rtol=0, atol=1e-15)


def test_topk_matches_sorting_with_ties_to_smaller_index():
    rng = np.random.default_rng(3)
    p = rng.integers(0, 6, (3, 50)).astype(np.float64)  # many ties
    for k in (1, 7, 25, 50):
        S = fo.select_topk(p, k)
        for h in range(3):
            ref = sorted(sorted(range(50), key=lambda j: (-p[h, j], j))[:k])
            assert list(S[h]) == ref


def _random_state(H=2, N=48, R=3, seed=5):
    rng = np.random.default_rng(seed)
    lay = fo.OracleLayer(H, R, 64)
    Kt = [None] + [rng.standard_normal((H, N, fo.HEAD_DIM)).astype(np.float32) for _ in range(R)]
    Vt = [None] + [rng.standard_normal((H, N, fo.HEAD_DIM)).astype(np.float32) for _ in range(R)]
    lay.set_tail(Kt, Vt, np.full(N, R))
    return lay, rng


def test_sparse_with_every_column_equals_dense():
    lay, rng = _random_state()
    q = [None] + [rng.standard_normal((2, fo.HEAD_DIM)).astype(np.float32) for _ in range(3)]
    lay.dense_loop(1, q[1])
    N = lay.n_cols
    S, m, u = lay.select(N)
    assert np.allclose(m, 1.0, atol=1e-12) and np.allclose(u, 0.0, atol=1e-12)
    sp = lay.sparse_loop(2, q[2], S)
    dense = fo.attention_dense(q[2], *lay.columns(2))[0]
    assert np.allclose(sp["o"], dense, rtol=1e-12, atol=1e-12)


def test_single_column_keeps_argmax_value_scaled_by_mass():
    lay, rng = _random_state()
    q = rng.standard_normal((2, fo.HEAD_DIM)).astype(np.float32)
    lay.dense_loop(1, q)
    p1 = lay.p_tilde.copy()
    S, m, u = lay.select(1)
    assert np.array_equal(S[:, 0], p1.argmax(axis=1))
    sp = lay.sparse_loop(2, q, S)
    V2 = lay.columns(2)[1]
    for h in range(2):
        assert np.allclose(sp["o"][h], u[h] + m[h] * V2[h, S[h, 0]], rtol=1e-12, atol=1e-12)


CODECS = [fo.RESIDUAL_INT4, fo.FULL_INT4, fo.RESIDUAL_INT2]


def _small_layer(seed=21, N=320, R=4, H=2, codec=fo.RESIDUAL_INT4):
    w = synth.Workload(name="t", layers=1, heads=H, n_ctx=N, loops=R,
                       sigma=(0, 0, 0.5, 0.2, 0.1)[:R + 1], frac=(0, 1, 1, 0.25, 0.10)[:R + 1], seed=seed)
    data = synth.prefill_layer(w, 0)
    sets = data["sets"]
    n_q, n_tail = synth.split_prefill(N)
    depth = synth.depth_of(sets, N).numpy()
    lay = fo.OracleLayer(H, R, 1024, codec=codec)
    f = lambda t: t.float().numpy()
    lay.encode_base(0, f(data["K"][1][:, :n_q]), f(data["V"][1][:, :n_q]))
    for r in range(2, R + 1):
        rows = sets[r][sets[r] < n_q].numpy()
        lay.encode_residual(r, rows, f(data["K"][r][:, rows]), f(data["V"][r][:, rows]))
    lay.set_tail([None] + [f(data["K"][r][:, n_q:]) for r in range(1, R + 1)],
                 [None] + [f(data["V"][r][:, n_q:]) for r in range(1, R + 1)], depth[n_q:])
    return w, data, lay, depth, n_q


@pytest.mark.parametrize("codec", CODECS)
def test_cache_invariants_nesting_and_inactive_reuse(codec):
    w, data, lay, depth, n_q = _small_layer(codec=codec)
    for r in range(2, w.loops + 1):
        inactive = np.nonzero(depth[:n_q] < r)[0]
        assert np.array_equal(lay.khat[r][:, inactive], lay.khat[r - 1][:, inactive])
        assert np.array_equal(lay.vhat[r][:, inactive], lay.vhat[r - 1][:, inactive])
        assert set(data["sets"][r].tolist()) <= set(data["sets"][r - 1].tolist())


def test_residual_is_taken_against_the_reconstruction():
    # With no change between loops the residual is exactly the loop-1 quantisation error,
    # so loop 2 must land much closer to the data than loop 1 (it would not move at all if
    # the residual were taken against the unquantised previous state).
    rng = np.random.default_rng(8)
    H, T = 2, 128
    X = torch.from_numpy(rng.standard_normal((H, T, fo.HEAD_DIM)).astype(np.float32)).bfloat16().float().numpy()
    lay = fo.OracleLayer(H, 2, T)
    lay.encode_base(0, X, X)
    lay.encode_residual(2, np.arange(T), X, X)
    e1 = np.abs(lay.khat[1][:, :T] - X).max()
    e2 = np.abs(lay.khat[2][:, :T] - X).max()
    assert e1 > 0 and e2 < e1 / 8


@pytest.mark.parametrize("codec", CODECS)
def test_full_schedule_invariants(codec):
    w, data, lay, depth, n_q = _small_layer(N=700, codec=codec)
    q = synth.queries(w, 0, 0).float().numpy()
    k_sel = w.k_sel(lay.n_cols)
    for r in range(1, w.loops + 1):
        if r <= w.dense_loops:
            out = lay.dense_loop(r, q[r])
        else:
            S, m, u = lay.select(k_sel)
            out = lay.sparse_loop(r, q[r], S)
            assert np.all((out["m"] >= 0) & (out["m"] <= 1 + 1e-12))
            assert np.allclose(out["m"], m) and np.allclose(out["u"], u)
        assert np.allclose(lay.p_tilde.sum(axis=1), 1.0, atol=1e-12)
        assert np.allclose(lay.output_identity(), out["o"], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("codec", CODECS)
def test_flush_moves_tail_into_the_base_and_residuals(codec):
    w, data, lay, depth, n_q = _small_layer(N=256, codec=codec)
    assert lay.n_tail == 64
    k_before = [lay.columns(r)[0].copy() for r in range(1, w.loops + 1)]
    step = synth.decode_token(w, 0, 0)
    lay.append_token([None] + [step["k"][r].float().numpy() for r in range(1, w.loops + 1)],
                     [None] + [step["v"][r].float().numpy() for r in range(1, w.loops + 1)])
    assert lay.n_q == n_q + 64 and lay.n_tail == 1
    for r in range(1, w.loops + 1):
        k_after = lay.columns(r)[0]
        old = k_before[r - 1]
        # flushed columns now carry quantisation error but stay close (half a 2-bit step
        # of a residual range is about twice half a 4-bit one); earlier columns unchanged
        assert np.array_equal(k_after[:, :n_q], old[:, :n_q])
        bound = 1.0 if codec == fo.RESIDUAL_INT2 else 0.5
        assert np.abs(k_after[:, n_q:n_q + 64] - old[:, n_q:n_q + 64]).max() < bound
        assert np.array_equal(k_after[:, -1], step["k"][r].float().numpy())

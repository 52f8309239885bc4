"""Pins for the oracle's token-sparse update selector.

Sources: FlashLoop project page, "The Method", Step 01 (only the tokens that stay
active are updated; inactive tokens reuse the preceding loop's state); flozi guide
"FlashLoop: store changes between repeated passes", section 3 (after the dense early
loops each loop ranks the previously updated tokens by normalized hidden-state change
and keeps a top-k subset; later selections are restricted to earlier active sets, so
the sets nest).

Each pin is fixed by the definition or by arithmetic done here independently (closed
forms with exact fp64 values, a Python-loop selection, invariants), so that a wrong
normalisation, a transposed pair of states, an inverted order, the wrong tie rule or a
selection that leaves the previous set fails one of them.
"""
import math

import numpy as np
import pytest

import synth
from oracle import flashloop_oracle as fo


def test_change_closed_forms():
    h_prev = np.zeros((5, 4))
    h_prev[:, :2] = [3.0, 4.0]                       # norm 5 on every row
    h_cur = h_prev.copy()
    h_cur[1] *= 2.0                                  # doubled: change = the state itself
    h_cur[2] += [1.0, 2.0, 2.0, 0.0]                 # change of norm 3
    h_cur[3] = -h_prev[3]                            # sign flip: change 2x the state
    h_cur[4] += [0.0, 0.0, 0.0, 5.0]                 # orthogonal change of the same norm
    key = fo.token_change(h_prev, h_cur)
    assert key.dtype == np.float64
    assert key.tolist() == [0.0, 1.0, 9.0 / 25.0, 4.0, 1.0]


def test_change_is_normalised_by_the_previous_state():
    rng = np.random.default_rng(7)
    hp = rng.standard_normal((6, 32)).astype(np.float32)
    hc = (hp + 0.3 * rng.standard_normal((6, 32))).astype(np.float32)
    key = fo.token_change(hp, hc)
    # scaling both states by a power of two leaves the relative change unchanged exactly
    assert np.array_equal(fo.token_change(hp * 8.0, hc * 8.0), key)
    # the definition restated with Python floats
    for j in range(6):
        num = math.fsum((float(c) - float(p)) ** 2 for p, c in zip(hp[j], hc[j]))
        den = math.fsum(float(p) ** 2 for p in hp[j])
        assert key[j] == pytest.approx(num / den, rel=1e-14)
    # swapping the two states changes the answer (the denominator is the earlier state)
    assert not np.allclose(fo.token_change(hc, hp), key)


def test_zero_previous_state():
    hp = np.zeros((3, 8))
    hc = np.zeros((3, 8))
    hc[1, 3] = 1.0
    key = fo.token_change(hp, hc)
    assert key[0] == 0.0 and key[2] == 0.0 and np.isinf(key[1]) and key[1] > 0


def _select_by_loop(key, rows, k):
    """k times: take the largest remaining key, the lowest token among equals."""
    left = list(zip(rows.tolist(), key.tolist()))
    out = []
    for _ in range(k):
        best = None
        for tok, kv in left:
            if best is None or kv > best[1] or (kv == best[1] and tok < best[0]):
                best = (tok, kv)
        out.append(best[0])
        left.remove(best)
    return sorted(out)


@pytest.mark.parametrize("n,k", [(1, 1), (9, 3), (40, 10), (40, 40), (40, 0)])
def test_select_matches_a_python_loop(n, k):
    rng = np.random.default_rng(n * 31 + k)
    hp = rng.standard_normal((n + 5, 16)).astype(np.float32)
    hc = (hp + rng.lognormal(size=(n + 5, 1)) * rng.standard_normal((n + 5, 16))).astype(np.float32)
    rows = np.sort(rng.choice(n + 5, size=n, replace=False))
    got = fo.select_active(hp, hc, rows, k)
    assert got.tolist() == _select_by_loop(fo.token_change(hp[rows], hc[rows]), rows, k)
    assert np.all(np.diff(got) > 0) and set(got.tolist()) <= set(rows.tolist())


def test_ties_go_to_the_lower_token_and_larger_changes_win():
    hp = np.ones((10, 4))
    hc = np.ones((10, 4)) * 1.5                      # every token changed by the same amount
    hc[7] = 3.0                                      # one token changed more
    hc[2] = 1.0                                      # one token did not change
    rows = np.arange(10)
    assert fo.select_active(hp, hc, rows, 1).tolist() == [7]
    assert fo.select_active(hp, hc, rows, 4).tolist() == [0, 1, 3, 7]
    assert 2 not in fo.select_active(hp, hc, rows, 9).tolist()
    assert fo.select_active(hp, hc, rows, 10).tolist() == list(range(10))


def test_nested_sets_from_hidden_states():
    w = synth.WORKLOADS["tiny_h1_n256"]
    n, d = 200, 64
    h = [t.float().numpy() for t in synth.hidden_states(w, n, d)]
    sizes = [0] + [w.n_active(r, n) for r in range(1, w.loops + 1)]
    sets = fo.nested_active_sets(h, sizes)
    assert sets[1].tolist() == list(range(n)) and sets[2].tolist() == list(range(n))
    for r in range(2, w.loops + 1):
        assert sets[r].size == sizes[r]
        assert set(sets[r].tolist()) <= set(sets[r - 1].tolist())
        assert np.all(np.diff(sets[r]) > 0)
    # loop 3 keeps the tokens that moved most in loop 2 (h[1] -> h[2]), among all tokens
    key = fo.token_change(h[1], h[2])
    kept, dropped = key[sets[3]], np.delete(key, sets[3])
    assert kept.min() >= dropped.max()
    # loop 4 ranks only loop 3's tokens, by their change in loop 3 (h[2] -> h[3])
    key4 = fo.token_change(h[2][sets[3]], h[3][sets[3]])
    in4 = np.isin(sets[3], sets[4])
    assert key4[in4].min() >= key4[~in4].max()

"""Token-sparse update selector (fl_select_active) against the oracle.

FlashLoop project page, "The Method", Step 01; flozi guide "FlashLoop: store changes
between repeated passes", section 3 (rank the previously updated tokens by normalized
hidden-state change, keep a top-k subset, nested sets).  Keys are fp64 on both sides
with different summation orders, so they agree to ~1e-15 relative; the selected sets
must be identical to the oracle's (and, independently of the oracle's ordering, a valid
top-k of the GPU's own keys with ties to the lower token).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import flashloop_oracle as fo
from quantized_kv_attention_int4_b200 import abi
from quantized_kv_attention_int4_b200.tokens import nested_active_sets

W = synth.WORKLOADS


def _run(hp, hc, rows, k, status=None):
    keys = torch.full((max(rows.numel(), 1),), -1.0, dtype=torch.float64, device="cuda")
    out = torch.full((max(k, 1),), -7, dtype=torch.int32, device="cuda")
    abi.fl_select_active(hp, hc, rows, k, out, keys, status=status)
    torch.cuda.synchronize()
    return out[:k].cpu().numpy(), keys[:rows.numel()].cpu().numpy()


def _valid_topk(keys, rows, out, k):
    sel = np.isin(rows, out)
    assert sel.sum() == k and np.all(np.diff(out) > 0)
    if 0 < k < rows.size:
        kin, kout = keys[sel], keys[~sel]
        assert kin.min() >= kout.max()
        # among equal keys at the boundary the lower tokens are the ones taken
        t = kin.min()
        if (kout == t).any():
            assert rows[sel & (keys == t)].max() < rows[~sel & (keys == t)].min()


@pytest.mark.gpu
@pytest.mark.parametrize("n,d,n_rows,k", [
    (1000, 256, 1000, 137), (1000, 256, 613, 1), (1000, 256, 613, 613), (4099, 2048, 3001, 1500),
    (77, 8, 50, 25), (5000, 1024, 0, 0), (300, 64, 300, 0)])
def test_select_matches_the_oracle(n, d, n_rows, k):
    w = W["tiny_h1_n256"]
    h = synth.hidden_states(w, n, d, device="cuda")
    g = torch.Generator().manual_seed(n + d + n_rows + k)
    rows = torch.sort(torch.randperm(n, generator=g)[:n_rows]).values.to(torch.int32).cuda()
    out, keys = _run(h[1], h[2], rows, k)
    r_np = rows.cpu().numpy().astype(np.int64)
    hp, hc = h[1].float().cpu().numpy(), h[2].float().cpu().numpy()
    ref_keys = fo.token_change(hp[r_np], hc[r_np])
    np.testing.assert_allclose(keys, ref_keys, rtol=1e-13, atol=0)
    assert out.tolist() == fo.select_active(hp, hc, r_np, k).tolist()
    _valid_topk(keys, r_np, out, k)


@pytest.mark.gpu
def test_ties_zero_states_and_row_stride():
    n, d = 600, 128
    base = torch.randn(n, d, dtype=torch.float32).to(torch.bfloat16)
    hp = torch.zeros(n, 256, dtype=torch.bfloat16)
    hc = torch.zeros(n, 256, dtype=torch.bfloat16)
    hp[:, :d] = base
    hc[:, :d] = (base.float() * 2).to(torch.bfloat16)          # every key exactly 1
    hp[5, :d] = 0                                               # zero state that changed: +inf
    hp[9, :d] = 0
    hc[9, :d] = 0                                               # zero state, no change: 0
    hc[:, d:] = 100.0                                           # beyond d_model: must be ignored
    hp_c, hc_c = hp.cuda()[:, :d], hc.cuda()[:, :d]             # row stride 256, d_model 128
    rows = torch.arange(n, dtype=torch.int32, device="cuda")
    out, keys = _run(hp_c, hc_c, rows, 40)
    assert np.isinf(keys[5]) and keys[9] == 0.0
    assert np.all(np.delete(keys, [5, 9]) == 1.0)
    assert out.tolist() == sorted([5] + [j for j in range(n) if j not in (5, 9)][:39])
    out_all, _ = _run(hp_c, hc_c, rows, n - 1)
    assert 9 not in out_all.tolist()


@pytest.mark.gpu
def test_bad_candidates_are_recorded_and_rank_last():
    n, d = 100, 64
    h = synth.hidden_states(W["tiny_h1_n256"], n, d, device="cuda")
    rows = torch.tensor([3, 10, 250, 40, 40, 77], dtype=torch.int32, device="cuda")
    status = torch.zeros(3, dtype=torch.int32, device="cuda")
    out, keys = _run(h[1], h[2], rows, 4, status)
    st = status.cpu().tolist()
    assert st[2] == 3 and st[0] in (abi.FL_DEV_ROWS_RANGE, abi.FL_DEV_ROWS_ORDER)  # 250; 40 after 250; 40 after 40
    assert np.isnan(keys[2])
    assert 250 not in out.tolist() and len(out) == 4


@pytest.mark.gpu
def test_nested_sets_at_full_size_match_the_oracle():
    w = W["cache_l48_h16_n32768"]
    n, d = w.n_ctx, 2048
    h = synth.hidden_states(w, n, d, device="cuda")
    sizes = [0] + [w.n_active(r, n) for r in range(1, w.loops + 1)]
    got = nested_active_sets(h, sizes)
    ref = fo.nested_active_sets([t.float().cpu().numpy() for t in h], sizes)
    for r in range(1, w.loops + 1):
        assert got[r].cpu().numpy().tolist() == ref[r].tolist(), r
    assert [t.numel() for t in got[1:]] == [n, n, 8192, 3277]


@pytest.mark.gpu
def test_cache_encoded_from_selected_sets_matches_the_oracle():
    from flhelpers import Pair, compare_encoding
    w = W["layer_h16_n4096"]
    h = synth.hidden_states(w, w.n_ctx, 256, device="cuda")
    sizes = [0] + [w.n_active(r, w.n_ctx) for r in range(1, w.loops + 1)]
    sets = [None] + [s.cpu().to(torch.int64) for s in nested_active_sets(h, sizes)[1:]]
    data = synth.prefill_layer(w, 0, device="cuda", sets=sets)
    pair = Pair(w, heads=[0, 9], data=data)
    compare_encoding(pair)

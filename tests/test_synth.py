"""Checks of the seeded input generators (shapes, nesting, determinism)."""
import torch

import synth


def test_split_prefill_keeps_a_1_to_64_row_tail():
    assert synth.split_prefill(256) == (192, 64)
    assert synth.split_prefill(4096) == (4032, 64)
    assert synth.split_prefill(32768) == (32704, 64)
    assert synth.split_prefill(8192) == (8128, 64)
    assert synth.split_prefill(65) == (64, 1)
    assert synth.split_prefill(1) == (0, 1)


def test_named_workload_set_sizes_and_key_budget():
    w = synth.WORKLOADS
    t = w["tiny_h1_n256"]
    assert [t.n_active(r, 256) for r in (1, 2, 3, 4)] == [256, 256, 64, 26] and t.k_sel(256) == 26
    l1 = w["layer_h16_n4096"]
    assert [l1.n_active(r, 4096) for r in (3, 4)] == [1024, 410] and l1.k_sel(4096) == 410
    l2 = w["layer_h16_n32768_decode256"]
    assert [l2.n_active(r, 32768) for r in (3, 4)] == [8192, 3277] and l2.k_sel(32768) == 3277
    d = w["deep_r32_h16_n8192"]
    assert d.loops == 32 and d.k_sel(8192) == 820
    assert abs(d.frac[2] - 0.9078) < 1e-3 and abs(d.frac[32] - 0.05) < 1e-12
    assert abs(d.sigma[4] - 0.5 * 0.85 ** 4) < 1e-15


def test_active_sets_nest_and_are_deterministic():
    w = synth.WORKLOADS["deep_r32_h16_n8192"]
    a = synth.active_sets(w, 1000)
    b = synth.active_sets(w, 1000)
    for r in range(1, w.loops + 1):
        assert torch.equal(a[r], b[r])
        assert a[r].numel() == w.n_active(r, 1000)
        if r > 1:
            assert set(a[r].tolist()) <= set(a[r - 1].tolist())
    d = synth.depth_of(a, 1000)
    for r in range(1, w.loops + 1):
        assert int((d >= r).sum()) == a[r].numel()


def test_prefill_changes_only_active_rows():
    w = synth.WORKLOADS["tiny_h1_n256"]
    x = synth.prefill_layer(w, 0)
    y = synth.prefill_layer(w, 0)
    for r in range(1, 5):
        assert torch.equal(x["K"][r], y["K"][r]) and x["K"][r].dtype == torch.bfloat16
    for r in range(2, 5):
        act = torch.zeros(256, dtype=torch.bool)
        act[x["sets"][r]] = True
        same = (x["K"][r] == x["K"][r - 1]).all(dim=2).all(dim=0)
        assert bool(same[~act].all()) and not bool(same[act].all())
    q = synth.queries(w, 0, 3)
    assert q.shape == (5, 1, 128) and not q[0].any()


def test_hidden_states_are_seeded_bf16_and_move_each_loop():
    w = synth.WORKLOADS["tiny_h1_n256"]
    a = synth.hidden_states(w, 50, 32)
    b = synth.hidden_states(w, 50, 32)
    assert len(a) == w.loops and all(t.dtype == torch.bfloat16 and t.shape == (50, 32) for t in a)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    for r in range(1, w.loops):
        assert not torch.equal(a[r], a[r - 1])

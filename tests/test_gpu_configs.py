"""The workload configurations end to end against the oracle, plus the launch patterns the
other parity tests do not reach.

* the 48-layer x 16-head 32K cache at the sizes, seeds and launch configuration bench.py
  times (one cache, the native loop-major executor), with sampled layers {0, 23, 47}
  checked loop by loop over a prompt-tail flush by the encoders, a decode step whose
  readers quantise the full tail (fused flush) and the step after it;
* the one-layer 32K cache through a prefill and 256 decode steps (five tail flushes),
  checked every 32 steps and around every flush, encodings bit-exact at the end;
* the 32-loop cache with every column selected, which needs more split-K partitions
  than the default 256 (the gather plan of each CTA must still fit its shared copy);
* standalone reader calls enqueued back to back with no host synchronisation between
  them, against the same calls synchronised one by one.

Tolerances as in the other parity tests: o, m and u within 2e-3 of the per-head
infinity norm of the fp64 oracle; the selected sets valid top-K up to 1e-5 max p~;
codes, scales and zeros bit-exact.
"""
import numpy as np
import pytest
import torch

import bench
import synth
from flhelpers import (TOL, Pair, check_topk_valid, compare_encoding, f32, note_elementwise, rel_err,
                       selection, u_err)
from oracle import flashloop_oracle as fo
from quantized_kv_attention_int4_b200 import abi
from quantized_kv_attention_int4_b200.cache import FlashLoopCache, round_up

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def _assert_errs(errs, tol=TOL):
    bad = {k: v for k, v in errs.items() if not (v <= tol)}
    assert not bad, bad


def test_full_cache_48_layers_sampled_layers_across_flushes():
    """The 48-layer cache (Ouro-2.6B-shaped: 48 layers x 16 heads x 128, 32K context, R = 4,
    per-layer seeds): the bench's own cache and executor."""
    w = W["cache_l48_h16_n32768"]
    L, R = w.layers, w.loops
    steps = 65
    device = torch.device("cuda")
    cache, wr = bench.build_cache(w, L, 0, device, new_tokens=steps)
    inputs = bench.step_inputs(wr, L, steps, device)
    step = bench.Step(cache, wr, L, device)
    layers, heads = (0, 23, 47), [3, 12]
    sets = synth.active_sets(wr, wr.n_ctx)
    oracles = {}
    for l in layers:
        d = synth.prefill_layer(wr, l, device="cuda", sets=sets)
        n_q, n_tail = synth.split_prefill(wr.n_ctx)
        lay = fo.OracleLayer(len(heads), R, cache.capacity)
        lay.encode_base(0, f32(d["K"][1][heads, :n_q]), f32(d["V"][1][heads, :n_q]))
        for r in range(2, R + 1):
            rows = sets[r][sets[r] < n_q].numpy()
            lay.encode_residual(r, rows, f32(d["K"][r][heads][:, rows]), f32(d["V"][r][heads][:, rows]))
        depth = synth.depth_of(sets, wr.n_ctx).numpy()
        lay.set_tail([None] + [f32(d["K"][r][heads, n_q:]) for r in range(1, R + 1)],
                     [None] + [f32(d["V"][r][heads, n_q:]) for r in range(1, R + 1)], depth[n_q:])
        oracles[l] = lay
        del d
    # step 0: the prompt's full tail is flushed by the encoders; step 63: the tail reaches
    # 64 rows and the step's readers quantise it; step 64: the first step after it
    checked = (0, 1, 62, 63, 64)
    fused_seen = False
    for s in range(steps):
        q, kn, vn = inputs[s]
        for l, lay in oracles.items():
            lay.append_token([None] + [f32(kn[r][l][heads]) for r in range(1, R + 1)],
                             [None] + [f32(vn[r][l][heads]) for r in range(1, R + 1)])
        if s not in checked:
            step.run(q, kn, vn)
            continue
        fused_seen |= cache.n_tail == 63      # this step's new token fills the tail
        step.run(q, kn, vn, loop_last=3)
        k_sel = wr.k_sel(cache.n_cols)
        S3 = {l: selection(cache, l, k_sel)[0] for l in layers}
        O123 = step.O[1:4].cpu().numpy()
        step.run(q, kn, vn, loop_first=4)
        O4 = step.O[4].cpu().numpy()
        for l, lay in oracles.items():
            errs = {}
            for r in (1, 2):
                ref = lay.dense_loop(r, f32(q[r][l][heads]))
                errs[(l, r)] = rel_err(O123[r - 1][l][heads], ref["o"])
                note_elementwise("cfg3 o", O123[r - 1][l][heads], ref["o"])
            check_topk_valid(S3[l][heads], lay.p_tilde, k_sel)
            ref = lay.sparse_loop(3, f32(q[3][l][heads]), S3[l][heads])
            errs[(l, 3)] = rel_err(O123[2][l][heads], ref["o"])
            o3_ref = ref["o"]
            S4, m4, u4 = selection(cache, l, k_sel)
            check_topk_valid(S4[heads], lay.p_tilde, k_sel)
            ref = lay.sparse_loop(4, f32(q[4][l][heads]), S4[heads])
            errs[(l, 4)] = rel_err(O4[l][heads], ref["o"])
            errs[(l, 4, "m")] = float(np.max(np.abs(m4[heads] - ref["m"]) / ref["m"]))
            errs[(l, 4, "u")] = u_err(u4[heads], ref["u"], O123[2][l][heads], o3_ref)
            note_elementwise("cfg3 o", O4[l][heads], ref["o"])
            note_elementwise("cfg3 u", u4[heads], ref["u"])
            _assert_errs(errs)
    assert fused_seen and cache.n_q == wr.n_ctx - 64 + 2 * 64 and cache.n_tail == 1
    st, info = cache.status()
    assert st == abi.FL_OK, info


def test_layer_32k_prefill_and_256_decode_steps():
    """One 16-head layer at 32K: prefill encode, then 256 decode
    steps through the step executor (the prompt's full tail flushed by the encoders at the
    first token, then a fused flush whenever the tail fills: steps 63, 127, 191, 255)."""
    w = W["layer_h16_n32768_decode256"]
    pair = Pair(w, heads=[3, 12], extra_tokens=256 + 64)
    compare_encoding(pair)
    checked = {0, 1, 255} | {s for s in range(256) if s % 32 == 0} | {63, 64, 127, 128, 191, 192}
    for step in range(256):
        tok = pair.begin_token(step)
        q = synth.queries(w, 0, step + 1, device="cuda")
        if step in checked:
            _assert_errs(pair.run_loops(q, tok, fused=True, label="cfg2"))
        else:
            pair.run_loops(q, tok, fused=True, oracle=False)
    assert pair.cache.n_q == 32704 + 5 * 64 and pair.cache.n_tail == 0
    # the oracle moves a full tail into its stores at the next append; the GPU's readers
    # did it inside step 255, so bring the oracle level before comparing the bytes
    assert pair.oracle.n_tail == 64
    pair.oracle.flush_tail()
    compare_encoding(pair)


def test_deep_loops_every_column_selected_needs_many_splits():
    """The 32-loop workload's shape (R = 32, N = 8192) with K_sel = N: a CTA of the
    loop > 8 reader holds at most 28 of the 36-word plan entries, so it needs ~293 split-K
    partitions per head (the loop <= 8 reader holds 56: ~147).  Every sparse loop must then
    equal the dense attention of its loop (m = 1)."""
    w = W["deep_r32_h16_n8192"]
    pair = Pair(w, heads=[0, 11])
    c = pair.cache
    N = c.n_cols
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n3, cap = abi.fl_sparse_splits(c.dims, 3, N, sms)
    n9, _ = abi.fl_sparse_splits(c.dims, 9, N, sms)
    assert 146 <= n3 <= cap and 256 < n9 <= cap
    q = synth.queries(w, 0, 0, device="cuda")
    errs = pair.run_loops(q, k_sel=N, label="deep K=N")
    # at K = N the unselected contribution is exactly zero in the oracle: hold u to the
    # output's scale there (every other entry keeps its own norm)
    u_errs = {k: v for k, v in errs.items() if isinstance(k, tuple) and k[1] == "u"}
    for k in u_errs:
        errs.pop(k)
    _assert_errs(errs)
    _, m, u = selection(c, 0, N)
    assert np.all(np.abs(m - 1) < 1e-5)
    assert np.abs(u).max() < 1e-4
    st, info = c.status()
    assert st == abi.FL_OK, info


def _cache_from(w, extra=80):
    n = w.n_ctx
    cap = round_up(n + extra + 64)
    cache = FlashLoopCache(1, w.heads, w.loops, cap, max_select=cap)
    d = synth.prefill_layer(w, 0, device="cuda")
    n_q, n_tail, tail_depth = cache.prefill_layer(0, d["K"], d["V"], d["sets"])
    cache.set_timeline(n_q, n_tail, tail_depth)
    return cache


def _standalone_steps(cache, w, steps, sync):
    """Decode `steps` tokens with the standalone entry points (k_new/v_new given to every
    reader), optionally synchronising after every call; returns each step's outputs."""
    H, R = w.heads, w.loops
    outs = []
    for s in range(steps):
        cache.begin_token()
        tok = synth.decode_token(w, 0, s, device="cuda")
        q = synth.queries(w, 0, s + 1, device="cuda")
        k = w.k_sel(cache.n_cols)
        O = torch.zeros(R + 1, H, 128, dtype=torch.float32, device="cuda")
        for r in range(1, R + 1):
            qr = q[r].contiguous()
            if r <= w.dense_loops:
                cache.dense(0, r, qr, O[r], tok["k"][r], tok["v"][r], keep_scores=True)
            else:
                if sync:
                    torch.cuda.synchronize()
                cache.select(0, 1, r, k)
                if sync:
                    torch.cuda.synchronize()
                cache.sparse(0, r, k, qr, O[r - 1], O[r], tok["k"][r], tok["v"][r])
            if sync:
                torch.cuda.synchronize()
        outs.append(O)
    torch.cuda.synchronize()
    return outs


def test_standalone_reader_calls_back_to_back_match_synchronised_calls():
    """A caller may chain the standalone reader entry points on one layer with nothing in
    between (each reader writes the new token's tail row and the layer's scores); the
    results must equal the same calls separated by host synchronisation, and the oracle."""
    w = W["layer_h16_n4096"]
    steps = 6
    a, b = _cache_from(w), _cache_from(w)
    out_a = _standalone_steps(a, w, steps, sync=False)
    out_b = _standalone_steps(b, w, steps, sync=True)
    for oa, ob in zip(out_a, out_b):
        assert np.array_equal(oa.cpu().numpy().view(np.uint32), ob.cpu().numpy().view(np.uint32))
    for name in ("score", "tag", "sel", "mass", "unsel", "tail_k", "tail_v"):
        assert torch.equal(a.raw(name, 0), b.raw(name, 0)), name
    # and the last step against the oracle (every loop), on a fresh pair of the same data
    pair = Pair(w, extra_tokens=80)
    for s in range(steps):
        tok = pair.begin_token(s)
        q = synth.queries(w, 0, s + 1, device="cuda")
        errs = pair.run_loops(q, tok, oracle=(s == steps - 1), label="standalone")
    _assert_errs(errs)
    for name in ("score", "tag", "mass", "unsel"):   # the pair issued the same calls
        assert torch.equal(a.raw(name, 0), pair.cache.raw(name, 0)), name
    for st in (a.status(), b.status()):
        assert st[0] == abi.FL_OK, st


@pytest.mark.parametrize("n_ctx", [60000, 100000])
def test_long_context_selection_through_thread_block_clusters(n_ctx):
    """Contexts beyond one CTA's shared memory (49152 columns): the selector spreads each
    (layer, head)'s keys over a cluster of 4 or 8 CTAs; S must still be a valid top-K of the
    oracle's distribution, and every loop must match the oracle."""
    w = synth.Workload(name=f"long{n_ctx}", layers=1, heads=2, n_ctx=n_ctx, loops=4,
                       sigma=(0, 0, 0.5, 0.2, 0.1), frac=(0, 1, 1, 0.25, 0.10), seed=31 + n_ctx)
    pair = Pair(w)
    errs = pair.run_loops(synth.queries(w, 0, 0, device="cuda"), label=f"N={n_ctx}")
    _assert_errs(errs)

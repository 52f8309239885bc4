"""GPU parity: the CUDA library against the oracle on the same seeded inputs.

Codes, scales and zero points must be bit-exact; attention outputs, the selected
mass m and the unselected contribution u within 2e-3 (max over heads of the
infinity-norm error divided by the reference's infinity norm); the selected set S
must be a valid top-K of the oracle's distribution (ties within 1e-5 of the
largest probability).  Sizes span several 64-token blocks and residual key groups
with ragged tails; the full-size cases use the launch configuration of bench.py
and check sampled heads.
"""
import numpy as np
import pytest
import torch

import synth
from flhelpers import TOL, Pair, compare_encoding, selection, rel_err, f32
from oracle import flashloop_oracle as fo
from quantized_kv_attention_int4_b200 import abi

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def _assert_errs(errs, tol=TOL):
    bad = {k: v for k, v in errs.items() if not (v <= tol)}
    assert not bad, bad


@pytest.mark.parametrize("name", ["tiny_h1_n256", "layer_h16_n4096"])
def test_prefill_encoding_is_bit_exact(name):
    pair = Pair(W[name])
    compare_encoding(pair)


@pytest.mark.parametrize("name", ["tiny_h1_n256", "layer_h16_n4096"])
def test_one_step_all_loops(name):
    w = W[name]
    pair = Pair(w)
    q = synth.queries(w, 0, 0, device="cuda")
    errs = pair.run_loops(q)
    _assert_errs(errs)


def test_ragged_prompt_lengths():
    # prompts whose tail is 1, 17 and 63 rows; quantised regions of 1..3 blocks
    for n in (65, 145, 255):
        w = synth.Workload(name=f"n{n}", layers=1, heads=3, n_ctx=n, loops=4,
                           sigma=(0, 0, 0.5, 0.2, 0.1), frac=(0, 1, 1, 0.25, 0.10), seed=77 + n)
        pair = Pair(w)
        compare_encoding(pair)
        _assert_errs(pair.run_loops(synth.queries(w, 0, 0, device="cuda")))


def test_tail_only_context():
    w = synth.Workload(name="n40", layers=1, heads=2, n_ctx=40, loops=4,
                       sigma=(0, 0, 0.5, 0.2, 0.1), frac=(0, 1, 1, 0.25, 0.10), seed=5)
    pair = Pair(w)
    assert pair.cache.n_q == 0
    _assert_errs(pair.run_loops(synth.queries(w, 0, 0, device="cuda")))


def test_full_retention_sparse_equals_dense():
    w = W["layer_h16_n4096"]
    pair = Pair(w)
    c, lay = pair.cache, pair.oracle
    q = synth.queries(w, 0, 0, device="cuda")
    N = c.n_cols
    o_prev = None
    for r in (1, 2):
        o = torch.empty(16, 128, device="cuda")
        c.dense(0, r, q[r].contiguous(), o, keep_scores=True)
        lay.dense_loop(r, f32(q[r]))
        o_prev = o
    c.select(0, 1, 3, N)
    S, _, _ = selection(c, 0, N)
    assert np.array_equal(S, np.tile(np.arange(N), (16, 1)))
    o = torch.empty(16, 128, device="cuda")
    c.sparse(0, 3, N, q[3].contiguous(), o_prev, o)
    _, m, u = selection(c, 0, N)
    assert np.all(np.abs(m - 1) < 1e-5)
    assert np.abs(u).max() < 1e-5 * np.abs(o_prev.cpu().numpy()).max() * 10
    ref = fo.attention_dense(f32(q[3]), *lay.columns(3))[0]
    assert rel_err(o.cpu().numpy(), ref) < TOL


def test_single_column_selection():
    w = W["layer_h16_n4096"]
    pair = Pair(w, heads=[0, 7])
    _assert_errs(pair.run_loops(synth.queries(w, 0, 1, device="cuda"), k_sel=1))


def test_decode_steps_across_two_flushes():
    w = W["tiny_h1_n256"]
    pair = Pair(w, extra_tokens=140)
    for step in range(130):
        tok = pair.begin_token(step)
        q = synth.queries(w, 0, step + 1, device="cuda")
        _assert_errs(pair.run_loops(q, tok))
    assert pair.cache.n_q == 192 + 3 * 64  # flushes at steps 0, 64 and 128
    compare_encoding(pair)


def test_decode_steps_multihead():
    w = W["layer_h16_n4096"]
    pair = Pair(w, heads=[1, 9, 15], extra_tokens=80)
    for step in range(70):
        tok = pair.begin_token(step)
        if step in (0, 1, 63, 64, 69):
            _assert_errs(pair.run_loops(synth.queries(w, 0, step + 1, device="cuda"), tok))
        else:
            pair.run_loops(synth.queries(w, 0, step + 1, device="cuda"), tok, check=False)
    compare_encoding(pair)


def test_deep_loops_r32():
    w = W["deep_r32_h16_n8192"]
    pair = Pair(w, heads=[0, 11])
    compare_encoding(pair)
    _assert_errs(pair.run_loops(synth.queries(w, 0, 0, device="cuda")))
    tok = pair.begin_token(0)
    _assert_errs(pair.run_loops(synth.queries(w, 0, 1, device="cuda"), tok))


def test_full_size_layer_32k_with_decode():
    w = W["layer_h16_n32768_decode256"]
    pair = Pair(w, heads=[3, 12], extra_tokens=70)
    compare_encoding(pair)
    for step in range(66):
        tok = pair.begin_token(step)
        if step in (0, 1, 65):
            _assert_errs(pair.run_loops(synth.queries(w, 0, step + 1, device="cuda"), tok))
        else:
            pair.run_loops(synth.queries(w, 0, step + 1, device="cuda"), tok, check=False)
    compare_encoding(pair)


def test_device_errors_are_recorded_not_trapped():
    w = synth.Workload(name="e", layers=1, heads=2, n_ctx=320, loops=4,
                       sigma=(0, 0, 0.5, 0.2, 0.1), frac=(0, 1, 1, 0.25, 0.10), seed=9)
    pair = Pair(w)
    c = pair.cache
    d = synth.prefill_layer(w, 0, device="cuda")
    assert c.status()[0] == abi.FL_OK
    # rows out of order
    rows = torch.tensor([10, 5], dtype=torch.int32, device="cuda")
    abi.fl_encode_residual(c.dims, c.buf, 0, 2, 0, 256, 320, rows, d["K"][2][:, :256],
                           d["V"][2][:, :256], compact=False)
    st, info = c.status()
    assert st == abi.FL_ERR_DEVICE and info[0] == 1 and info[1] == 5
    # loop-4 row that is not active in loop 3
    inactive3 = int(np.setdiff1d(np.arange(256), pair.sets[3].numpy())[0])
    rows = torch.tensor([inactive3], dtype=torch.int32, device="cuda")
    abi.fl_encode_residual(c.dims, c.buf, 0, 4, 0, 256, 320, rows, d["K"][4][:, :256], d["V"][4][:, :256],
                           compact=False)
    st, info = c.status()
    assert st == abi.FL_ERR_DEVICE and info[0] == 3 and info[1] == inactive3
    # a selected column out of range is skipped and reported (on a fresh, consistent cache)
    pair = Pair(w)
    c = pair.cache
    q = synth.queries(w, 0, 0, device="cuda")
    o = torch.empty(2, 128, device="cuda")
    c.dense(0, 1, q[1].contiguous(), o, keep_scores=True)
    c.select(0, 1, 2, 10)
    ps = c.layout.plan_stride
    c.raw("plan", 0).view(torch.int32)[3 * ps] = 100000   # head 0, fourth selected column
    o2 = torch.empty(2, 128, device="cuda")
    c.sparse(0, 2, 10, q[2].contiguous(), o, o2)
    st, info = c.status()
    assert st == abi.FL_ERR_DEVICE and info[0] == 4 and info[1] == 100000
    assert torch.isfinite(o2).all()


@pytest.mark.parametrize("name", ["tiny_h1_n256", "layer_h16_n4096"])
def test_dense_reader_at_every_loop(name):
    """The dense reader at loops 1..R (loops 1-3: the staged form with up to two residual
    stores; deeper loops: the direct form) against the oracle's full attention, with the
    kept scores reproducing the oracle's log-probabilities."""
    w = W[name]
    pair = Pair(w)
    c, lay = pair.cache, pair.oracle
    q = synth.queries(w, 0, 0, device="cuda")
    H, N = w.heads, c.n_cols
    for r in range(1, w.loops + 1):
        o = torch.empty(H, 128, dtype=torch.float32, device="cuda")
        c.dense(0, r, q[r].contiguous(), o, keep_scores=True)
        ref = lay.dense_loop(r, f32(q[r]))
        assert rel_err(o.cpu().numpy(), ref["o"]) < TOL, r
        sc = c.raw("score", 0).view(torch.float32)[: H * c.dims.capacity].view(H, -1)[:, :N].cpu().numpy()
        off = c.raw("offset", 0).view(torch.float32)[: H * 33].view(H, 33)[:, r].cpu().numpy()
        lp = sc.astype(np.float64) - off[:, None]
        assert np.abs(lp - np.log2(ref["p"])).max() < 1e-4, r
    st, info = c.status()
    assert st == abi.FL_OK, info

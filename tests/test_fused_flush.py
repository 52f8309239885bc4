"""Fused tail flush (fl_decode_step_flush): a decode step whose BF16 tail holds 64 rows
also writes that tail's INT4 stores from inside its readers (FlashLoop project page,
"The Method", closing paragraph: KV updates and quantisation fused into attention).

* The step's outputs are bit-identical to the same step without the flush.
* The base / residual records, masks, first slots and depths it writes are
  bit-identical to those of the separate encode launches (fl_encode_base /
  fl_encode_residual) on the same rows, for dense and sparse loops, the staged and the
  direct readers, a new token in tail row 63 or a prompt tail without one.
* Decoding across several fused flushes matches the oracle loop by loop, and the
  final encoding is the oracle's.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from flhelpers import TOL, Pair, compare_encoding
from quantized_kv_attention_int4_b200 import abi
from quantized_kv_attention_int4_b200.cache import FlashLoopCache, round_up

W = synth.WORKLOADS
STORES = ("brec", "rrec", "mask", "first", "depth")


def _build(w, layers, extra=130):
    n = w.n_ctx
    cap = round_up(n + extra + 64)
    sets = synth.active_sets(w, n)
    cache = FlashLoopCache(layers, w.heads, w.loops, cap, max_select=cap)
    info = None
    for layer in range(layers):
        d = synth.prefill_layer(w, layer, device="cuda", sets=sets)
        info = cache.prefill_layer(layer, d["K"], d["V"], sets)
        del d
    cache.set_timeline(*info)
    return cache


def _inputs(w, layers, step):
    """q, k_new, v_new as [R+1][L][H][128] BF16 for decode step ``step``."""
    R = w.loops
    zero = torch.zeros(w.heads, 128, dtype=torch.bfloat16, device="cuda")
    q = torch.stack([synth.queries(w, layer, step, device="cuda") for layer in range(layers)], dim=1)
    toks = [synth.decode_token(w, layer, step, device="cuda") for layer in range(layers)]
    kn = torch.stack([torch.stack([zero] + t["k"][1:]) for t in toks], dim=1)
    vn = torch.stack([torch.stack([zero] + t["v"][1:]) for t in toks], dim=1)
    assert kn.shape == (R + 1, layers, w.heads, 128)
    return q.contiguous(), kn.contiguous(), vn.contiguous()


def _run(cache, w, step, new_token=True, flush=False):
    q, kn, vn = _inputs(w, cache.L, step)
    O = torch.zeros(w.loops + 1, cache.L, w.heads, 128, dtype=torch.float32, device="cuda")
    cache.step(w.dense_loops, w.k_sel(cache.n_cols), q, O, kn if new_token else None, vn if new_token else None,
               flush=flush)
    st, info = cache.status()
    assert st == abi.FL_OK, info
    return O[1:].cpu().numpy()


def _bits_equal(a, b):
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def _same_stores(a, b):
    for layer in range(a.L):
        for name in STORES:
            assert torch.equal(a.raw(name, layer), b.raw(name, layer)), (layer, name)


@pytest.mark.gpu
@pytest.mark.parametrize("base,layers,dense_loops", [
    ("layer_h16_n4096", 2, 2),      # dense staged loops 1-2, sparse staged loops 3-4
    ("layer_h16_n4096", 2, 4),      # every loop dense (loop 4 on the direct reader)
    ("deep_r32_h16_n8192", 2, 5),   # dense direct loops 4-5, sparse staged 6-8, sparse direct 9-32
])
def test_fused_flush_of_a_decoded_tail_matches_the_encoders(base, layers, dense_loops):
    w0 = W[base]
    w = dataclasses.replace(w0, name=w0.name + "_tail63", n_ctx=w0.n_ctx - 1, dense_loops=dense_loops)
    A, B = _build(w, layers), _build(w, layers)
    assert A.n_tail == 63
    A.begin_token()
    B.begin_token()
    oa = _run(A, w, 0)
    ob = _run(B, w, 0, flush=True)          # tail row 63 is the new token (k_new / v_new)
    _bits_equal(oa, ob)
    assert B.n_tail == 0 and B.n_q == A.n_q + 64
    A.begin_token()                          # A's full tail goes through the encode launches here
    B.begin_token()
    assert (A.n_q, A.n_tail, A.tail_depth) == (B.n_q, B.n_tail, B.tail_depth)
    assert A.n_slots == B.n_slots and A.n_rows == B.n_rows
    _same_stores(A, B)
    _bits_equal(_run(A, w, 1), _run(B, w, 1))


@pytest.mark.gpu
def test_fused_flush_of_a_prompt_tail_matches_the_encoders():
    w = W["layer_h16_n4096"]                 # 4096 prompt columns: a full tail of prompt rows
    A, B = _build(w, 2), _build(w, 2)
    assert A.n_tail == 64 and len(set(A.tail_depth)) > 1
    oa = _run(A, w, 0, new_token=False)
    ob = _run(B, w, 0, new_token=False, flush=True)
    _bits_equal(oa, ob)
    A.begin_token()
    B.begin_token()
    assert A.n_slots == B.n_slots
    _same_stores(A, B)


@pytest.mark.gpu
def test_flush_plan_is_validated_on_the_host():
    w = W["tiny_h1_n256"]
    c = _build(w, 1, extra=0)
    q, kn, vn = _inputs(w, 1, 0)
    O = torch.zeros(w.loops + 1, 1, w.heads, 128, dtype=torch.float32, device="cuda")
    k = w.k_sel(c.n_cols)
    good = c.flush_plan()

    def call(plan, n_tail=64):
        abi.fl_decode_step(c.dims, c.buf, c.n_q, n_tail, w.dense_loops, k, 1, w.loops, q, None, None, O, c.ws,
                           flush=plan)

    bad_nest = abi.Flush([0, 0, 0b01, 0b11, 0], [[0] * 5])
    with pytest.raises(abi.FlashLoopError):
        call(bad_nest)                       # loop 3's rows are not inside loop 2's
    bad_slot = abi.Flush(list(good.active), [[0, 0, 32, 0, 0]])
    with pytest.raises(abi.FlashLoopError):
        call(bad_slot)                       # not a multiple of 64
    full = abi.Flush(list(good.active), [[0, 0, c.capacity, c.capacity, c.capacity]])
    with pytest.raises(abi.FlashLoopError):
        call(full)                           # past the store's capacity
    with pytest.raises(abi.FlashLoopError):
        call(good, n_tail=63)                # only a full tail can be flushed


def _decode(pair, steps, check_at=None):
    w = pair.w
    for step in range(steps):
        tok = pair.begin_token(step)
        q = synth.queries(w, 0, step + 1, device="cuda")
        if check_at is None or step in check_at:
            errs = pair.run_loops(q, tok, fused=True)
            bad = {k: v for k, v in errs.items() if not v < TOL}
            assert not bad, (step, bad)
        else:
            pair.run_loops(q, tok, fused=True, check=False)


@pytest.mark.gpu
def test_decode_across_three_fused_flushes_matches_the_oracle():
    w0 = W["tiny_h1_n256"]
    w = dataclasses.replace(w0, name="tiny_h1_n255", n_ctx=255)
    pair = Pair(w, extra_tokens=140)
    _decode(pair, 130)
    assert pair.cache.n_q == 192 + 3 * 64    # flushed inside steps 0, 64 and 128
    compare_encoding(pair)


@pytest.mark.gpu
def test_decode_multihead_fused_flush_matches_the_oracle():
    w0 = W["layer_h16_n4096"]
    w = dataclasses.replace(w0, name="layer_h16_n4095", n_ctx=4095)
    pair = Pair(w, heads=[0, 6, 15], extra_tokens=80)
    _decode(pair, 66, check_at=(0, 1, 64, 65))
    compare_encoding(pair)

"""GPU parity of the codec variants of the loop r >= 2 stores.

flozi guide "FlashLoop: store changes between repeated passes", section 4: the
"Per-loop KIVI4" ablation (full KV states quantised per loop) and the 2-bit residual
row of Figure 5; FlashLoop project page, "Experiments", caption of Figure 5 (residual
precision varied with the other components fixed).

The library's encoders must write the oracle's codes, scales and zero points bit for
bit (2-bit codes unpacked from the 5120-byte records by the test's own reader of the
documented layout); dense and sparse loops, through the per-loop entry points and
the step executor, must match the oracle within 2e-3, on prompts with ragged tails,
loop-2 sets smaller than the context (so the full-state base is read for some tokens
and skipped for others), every loop dense, and 32 loops.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from flhelpers import TOL, Pair, compare_encoding
from quantized_kv_attention_int4_b200 import abi

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CODECS = [abi.FL_CODEC_FULL_INT4, abi.FL_CODEC_RESIDUAL_INT2]
IDS = {abi.FL_CODEC_FULL_INT4: "full4", abi.FL_CODEC_RESIDUAL_INT2: "res2"}


def _ok(errs, tol=TOL):
    bad = {k: v for k, v in errs.items() if not (v <= tol)}
    assert not bad, bad


def _partial_loop2(name="n1000_part", n=1000, heads=4, seed=91):
    # loop 2 updates 60 % of the tokens: full-state blocks mix base and loop-2 rows
    return synth.Workload(name=name, layers=1, heads=heads, n_ctx=n, loops=4,
                          sigma=(0, 0, 0.5, 0.2, 0.1), frac=(0, 1, 0.6, 0.25, 0.10), seed=seed)


@pytest.mark.parametrize("codec", CODECS, ids=IDS.get)
@pytest.mark.parametrize("name", ["tiny_h1_n256", "layer_h16_n4096", "partial"])
def test_variant_encoding_is_bit_exact(codec, name):
    w = _partial_loop2() if name == "partial" else W[name]
    pair = Pair(w, heads=[0, 5, 15] if w.heads == 16 else None, codec=codec)
    compare_encoding(pair)


@pytest.mark.parametrize("codec", CODECS, ids=IDS.get)
@pytest.mark.parametrize("name,dense_loops", [
    ("tiny_h1_n256", 2), ("layer_h16_n4096", 2), ("partial", 2), ("partial", 4), ("ragged", 2), ("ragged", 4),
])
def test_variant_loops_match_the_oracle(codec, name, dense_loops):
    if name == "partial":
        w = _partial_loop2()
    elif name == "ragged":
        w = _partial_loop2("n145_part", 145, 3, 92)       # two quantised blocks plus a 17-row tail
    else:
        w = W[name]
    w = dataclasses.replace(w, dense_loops=dense_loops)
    pair = Pair(w, heads=[0, 7, 15] if w.heads == 16 else None, codec=codec)
    tok = pair.begin_token(0)
    _ok(pair.run_loops(synth.queries(w, 0, 1, device="cuda"), tok))


@pytest.mark.parametrize("codec", CODECS, ids=IDS.get)
def test_variant_32_loops(codec):
    w = W["deep_r32_h16_n8192"]
    pair = Pair(w, heads=[0, 9], codec=codec)
    compare_encoding(pair)
    _ok(pair.run_loops(synth.queries(w, 0, 0, device="cuda")))


@pytest.mark.parametrize("codec", CODECS, ids=IDS.get)
def test_variant_decode_across_a_flush_and_the_executor(codec):
    w = dataclasses.replace(W["tiny_h1_n256"], name="tiny_h1_n255", n_ctx=255)
    pair = Pair(w, extra_tokens=70, codec=codec)
    for step in range(66):
        tok = pair.begin_token(step)           # step 1 flushes the full tail through the encoders
        q = synth.queries(w, 0, step + 1, device="cuda")
        fused = step % 2 == 1                  # odd steps run through fl_decode_step (no tail flush)
        if step in (0, 1, 2, 64, 65):
            _ok(pair.run_loops(q, tok, fused=fused))
        else:
            pair.run_loops(q, tok, fused=fused, check=False)
    assert pair.cache.n_q == 320                # flushed at the appends of steps 1 and 65
    compare_encoding(pair)


@pytest.mark.parametrize("codec", CODECS, ids=IDS.get)
def test_fused_flush_is_refused_for_variants(codec):
    w = W["tiny_h1_n256"]
    pair = Pair(w, codec=codec)
    c = pair.cache
    assert c.n_tail == 64
    q = synth.queries(w, 0, 0, device="cuda")[:, None].contiguous()
    O = torch.zeros(w.loops + 1, 1, w.heads, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(abi.FlashLoopError) as e:
        c.step(w.dense_loops, w.k_sel(c.n_cols), q, O, flush=True)
    assert e.value.status == abi.FL_ERR_UNSUPPORTED
    st, info = c.status()
    assert st == abi.FL_OK, info


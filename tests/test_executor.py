"""The native step executor (fl_decode_step: loop-major over layers, selection for all
layers in one launch, readers launched back to back) against the oracle, layer by layer
and loop by loop, on a two-layer cache; and a whole step in one call reproducing the
loop-by-loop bytes."""
import numpy as np
import pytest
import torch

import synth
from flhelpers import TOL, check_topk_valid, f32, rel_err, selection
from oracle import flashloop_oracle as fo
from quantized_kv_attention_int4_b200 import abi
from quantized_kv_attention_int4_b200.cache import FlashLoopCache, round_up

W = synth.WORKLOADS


def _build(w, layers):
    n = w.n_ctx
    cap = round_up(n + 128)
    sets = synth.active_sets(w, n)
    cache = FlashLoopCache(layers, w.heads, w.loops, cap, max_select=cap)
    oracles = []
    info = None
    for layer in range(layers):
        d = synth.prefill_layer(w, layer, device="cuda", sets=sets)
        info = cache.prefill_layer(layer, d["K"], d["V"], sets)
        n_q, n_tail, tail_depth = info
        lay = fo.OracleLayer(w.heads, w.loops, cap)
        lay.encode_base(0, f32(d["K"][1][:, :n_q]), f32(d["V"][1][:, :n_q]))
        for r in range(2, w.loops + 1):
            rows = sets[r][sets[r] < n_q].numpy()
            lay.encode_residual(r, rows, f32(d["K"][r][:, rows]), f32(d["V"][r][:, rows]))
        lay.set_tail([None] + [f32(d["K"][r][:, n_q:]) for r in range(1, w.loops + 1)],
                     [None] + [f32(d["V"][r][:, n_q:]) for r in range(1, w.loops + 1)], np.array(tail_depth))
        oracles.append(lay)
    cache.set_timeline(*info)
    return cache, oracles


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny_h1_n256", "layer_h16_n4096"])
def test_native_step_executor_matches_the_oracle(name):
    w = W[name]
    L, R, H = 2, w.loops, w.heads
    cache, oracles = _build(w, L)
    q = torch.stack([synth.queries(w, layer, 0, device="cuda") for layer in range(L)], dim=1).contiguous()
    O = torch.zeros(R + 1, L, H, 128, dtype=torch.float32, device="cuda")
    k = w.k_sel(cache.n_cols)
    for r in range(1, R + 1):
        cache.step(w.dense_loops, k, q, O, loop_first=r, loop_last=r)
        got = O[r].cpu().numpy()
        for layer in range(L):
            lay = oracles[layer]
            if r <= w.dense_loops:
                ref = lay.dense_loop(r, f32(q[r][layer]))["o"]
            else:
                S, _, _ = selection(cache, layer, k)
                check_topk_valid(S, lay.p_tilde, k)
                ref = lay.sparse_loop(r, f32(q[r][layer]), S)["o"]
            assert rel_err(got[layer], ref) < TOL, (r, layer)
    st, info = cache.status()
    assert st == abi.FL_OK, info

    # the whole step in one call (loop 1 rewrites every score, so the state repeats)
    O2 = torch.zeros_like(O)
    cache.step(w.dense_loops, k, q, O2)
    torch.cuda.synchronize()
    assert np.array_equal(O2[1:].cpu().numpy().view(np.uint32), O[1:].cpu().numpy().view(np.uint32))

"""The sparse reader's no-workspace entry point (library-owned static scratch) gives the
same bytes as the workspace entry point, on two calls in a row -- on the staged reader
(loops <= 8) and on the direct one (loops 9 and 10 of the 32-loop cache), whose split
counts differ.

Kept in a file collected last so that it also runs after every other GPU test has used
the library (the static scratch keeps its contents between calls)."""
import numpy as np
import pytest
import torch

import synth
from flhelpers import Pair
from quantized_kv_attention_int4_b200 import abi

W = synth.WORKLOADS


@pytest.mark.gpu
@pytest.mark.parametrize("name,loops", [("tiny_h1_n256", (3, 4)), ("layer_h16_n4096", (3, 4)),
                                        ("deep_r32_h16_n8192", (3, 9, 10))])
def test_noalloc_sparse_matches_workspace_call(name, loops):
    w = W[name]
    pair = Pair(w)
    c = pair.cache
    q = synth.queries(w, 0, 0, device="cuda")
    k = w.k_sel(c.n_cols)
    H = w.heads
    o_prev = None
    for r in range(1, w.dense_loops + 1):
        o = torch.empty(H, 128, dtype=torch.float32, device="cuda")
        c.dense(0, r, q[r].contiguous(), o, keep_scores=True)
        o_prev = o
    for r in loops:
        c.select(0, 1, r, k)
        qr = q[r].contiguous()
        o_ws = torch.empty(H, 128, dtype=torch.float32, device="cuda")
        c.sparse(0, r, k, qr, o_prev, o_ws)
        outs = []
        for _ in range(2):
            o_na = torch.full((H, 128), float("nan"), dtype=torch.float32, device="cuda")
            abi.fl_decode_attn_sparse_noalloc(c.dims, c.buf, 0, r, c.n_q, c.n_tail, k, qr, None, None, o_prev, o_na)
            outs.append(o_na)
        torch.cuda.synchronize()
        ref = o_ws.cpu().numpy()
        assert np.all(np.isfinite(ref))
        for o_na in outs:
            assert np.array_equal(o_na.cpu().numpy().view(np.uint32), ref.view(np.uint32))
        o_prev = o_ws
    st, info = c.status()
    assert st == abi.FL_OK, info

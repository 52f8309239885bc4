"""The executor's outputs are a function of its inputs alone: two caches built the same
way give bit-identical outputs for every loop of a decode step.  The persistent sparse
reader hands each batch from warp to warp through shared memory and reuses an item's
plan slot for its final merge; a hand-off that raced would show here as outputs that
differ between two runs (the oracle comparisons would only see it as noise within their
tolerance).  Configurations: loops 3-4 over items of several batches (4096 columns), and
loops 6-32 of the 32-loop cache, whose items of 56 columns are mostly one batch each.
"""
import dataclasses

import numpy as np
import pytest

import synth
from test_fused_flush import _build, _run

W = synth.WORKLOADS


@pytest.mark.gpu
@pytest.mark.parametrize("base,dense_loops", [("layer_h16_n4096", 2), ("deep_r32_h16_n8192", 5)])
def test_two_identical_caches_give_identical_outputs(base, dense_loops):
    w = dataclasses.replace(W[base], dense_loops=dense_loops)
    A, B = _build(w, 2), _build(w, 2)
    for step in range(2):
        A.begin_token()
        B.begin_token()
        oa, ob = _run(A, w, step), _run(B, w, step)
        for r in range(oa.shape[0]):
            assert np.array_equal(oa[r].view(np.uint32), ob[r].view(np.uint32)), (step, r + 1)

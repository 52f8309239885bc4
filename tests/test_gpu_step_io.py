"""fl_decode_step_io: the executor fed from and returning to host memory in one call (the
input copy runs beside the first loop's selection on the library's copy stream) gives
outputs bit-identical to the same step fed from device memory, for whole steps, for a
step's later loops alone, and for a step whose readers quantise a full tail."""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from test_fused_flush import _build, _inputs

W = synth.WORKLOADS


def _device_step(c, w, step, flush, loop_first=1, loop_last=None, O=None):
    q, kn, vn = _inputs(w, c.L, step)
    if O is None:
        O = torch.zeros(w.loops + 1, c.L, w.heads, 128, dtype=torch.float32, device="cuda")
    c.step(w.dense_loops, w.k_sel(c.n_cols), q, O, kn, vn, loop_first=loop_first, loop_last=loop_last or w.loops,
           flush=flush)
    return O


def _host_step(c, w, step, flush, loop_first=1, loop_last=None, O=None):
    R = w.loops
    loop_last = loop_last or R
    q, kn, vn = _inputs(w, c.L, step)
    if O is None:
        O = torch.zeros(R + 1, c.L, w.heads, 128, dtype=torch.float32, device="cuda")
    qkv = torch.zeros(3, R + 1, c.L, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    # loops before loop_first were run from device memory (their inputs are in place)
    for i, t in enumerate((q, kn, vn)):
        qkv[i, :loop_first] = t[:loop_first]
    sl = slice(loop_first, loop_last + 1)
    host_in = torch.stack([q[sl], kn[sl], vn[sl]]).cpu().pin_memory()
    host_out = torch.zeros(loop_last - loop_first + 1, c.L, w.heads, 128, dtype=torch.float32).pin_memory()
    c.step_io(w.dense_loops, w.k_sel(c.n_cols), qkv, host_in, O, host_out, loop_first=loop_first,
              loop_last=loop_last, flush=flush)
    torch.cuda.synchronize()
    assert torch.equal(host_out, O[sl].cpu())
    return O


def _same(a, b):
    a, b = a.cpu().numpy(), b.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.gpu
def test_host_buffers_match_device_buffers_over_steps_and_a_flush():
    w0 = W["layer_h16_n4096"]
    w = dataclasses.replace(w0, name=w0.name + "_tail63", n_ctx=w0.n_ctx - 1)
    A, B = _build(w, 2), _build(w, 2)
    for step in range(3):
        A.begin_token()
        B.begin_token()
        flush = A.n_tail == 64                   # the first step's tail is full: fused flush
        _same(_device_step(A, w, step, flush), _host_step(B, w, step, flush))


@pytest.mark.gpu
def test_host_buffers_for_the_late_loops_of_a_step():
    w = W["layer_h16_n4096"]
    A, B = _build(w, 2), _build(w, 2)
    A.begin_token()
    B.begin_token()
    OA = _device_step(A, w, 0, False, loop_first=1, loop_last=2)
    OB = _device_step(B, w, 0, False, loop_first=1, loop_last=2)
    _same(_device_step(A, w, 0, False, loop_first=3, O=OA), _host_step(B, w, 0, False, loop_first=3, O=OB))

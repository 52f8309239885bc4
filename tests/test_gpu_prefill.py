"""Sparse prefill attention on the tensor cores (fl_prefill_attn_sparse) against the
oracle.

FlashLoop project page, "The Method", Step 01 (only the active tokens are recomputed)
and the paragraph after Step 03 (selected tokens gathered into compact buffers so the
work stays a regular GEMM).  Tolerance, from the arithmetic: the kernel rounds each
probability to BF16 (relative error <= 2^-9) before the value product and normalises by
the fp32 sum of the unrounded ones, so |o - o_ref| <= 2^-9 * sum_j p_j |v_j| / sum_j p_j
<= 2^-9 max|v| per head, plus fp32 accumulation; the test allows 2^-8 max|v|.
"""
import numpy as np
import pytest
import torch

from oracle import flashloop_oracle as fo
from quantized_kv_attention_int4_b200 import abi


def _inputs(H, N, pos, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    k = torch.randn(H, N, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(H, N, 128, generator=g).to(torch.bfloat16)
    q = torch.randn(H, len(pos), 128, generator=g).to(torch.bfloat16)
    return q, k, v


def _run(q, pos, k, v, status=None, fill=0.0):
    o = torch.full((q.shape[0], q.shape[1], 128), fill, dtype=torch.float32, device="cuda")
    abi.fl_prefill_attn_sparse(q.cuda(), torch.as_tensor(pos, dtype=torch.int32).cuda(), k.cuda(), v.cuda(), o,
                               status=status)
    torch.cuda.synchronize()
    return o.cpu().numpy()


def _check(q, pos, k, v, o):
    ref = fo.prefill_attention(q.float().numpy(), np.asarray(pos), k.float().numpy(), v.float().numpy())
    bound = 2.0 ** -8 * np.abs(v.float().numpy()).max(axis=(1, 2))
    err = np.abs(o - ref).max(axis=(1, 2))
    assert np.all(err <= bound), (err, bound)
    return err


@pytest.mark.gpu
@pytest.mark.parametrize("H,N,n_act,seed", [
    (2, 300, 100, 1), (1, 256, 256, 2), (3, 1000, 130, 3), (1, 77, 1, 4), (4, 4096, 1024, 5), (2, 129, 129, 6)])
def test_prefill_matches_the_oracle(H, N, n_act, seed):
    rng = np.random.default_rng(seed)
    pos = np.sort(rng.choice(N, size=n_act, replace=False))
    if n_act == 1:
        pos = np.array([N - 1])
    q, k, v = _inputs(H, N, pos, seed)
    _check(q, pos, k, v, _run(q, pos, k, v))


@pytest.mark.gpu
def test_all_active_equals_causal_attention():
    H, N = 2, 512
    q, k, v = _inputs(H, N, np.arange(N), 7)
    o = _run(q, np.arange(N), k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(), is_causal=True)
    bound = 2.0 ** -8 * v.float().abs().amax(dim=(1, 2)).numpy()
    assert np.all(np.abs(o - ref.numpy()).max(axis=(1, 2)) <= bound)


@pytest.mark.gpu
def test_bad_positions_are_recorded_and_left_unwritten():
    H, N = 1, 400
    pos = np.array([3, 50, 999, 60, 300])      # 999 out of range; 60 after 999 is out of order
    q, k, v = _inputs(H, N, pos, 8)
    status = torch.zeros(3, dtype=torch.int32, device="cuda")
    o = _run(q, pos, k, v, status=status, fill=7.0)
    st = status.cpu().tolist()
    assert st[2] == 2 and st[0] in (abi.FL_DEV_ROWS_RANGE, abi.FL_DEV_ROWS_ORDER)
    assert np.all(o[0, 2] == 7.0)
    good = [0, 1, 3, 4]
    ref = fo.prefill_attention(q.float().numpy()[:, good], pos[good], k.float().numpy(), v.float().numpy())
    assert np.abs(o[:, good] - ref).max() <= 2.0 ** -8 * np.abs(v.float().numpy()).max()

"""The C-ABI library loads on a machine without a GPU, exports every symbol the header
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

from quantized_kv_attention_int4_b200 import abi
from quantized_kv_attention_int4_b200.cache import round_up, split_prefill

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "flashloop.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:fl_status|size_t|const char\*)\s+(fl_\w+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) == 20
    for n in names:
        assert hasattr(abi.lib, n), n
    assert set(names) == set(abi.EXPORTED)
    assert "sm_100a" in abi.fl_version()


def _dims(**kw):
    base = dict(layers=2, heads=4, loops=4, capacity=1024, max_select=128,
                res_capacity={2: 1024, 3: 256, 4: 128})
    base.update(kw)
    return abi.Dims(**base)


def test_layout_is_aligned_and_consistent():
    d = _dims()
    L = abi.fl_cache_layout(d)
    offs = [getattr(L, n) for n in abi.ARRAY_NAMES] + [L.status]
    assert L.plan_stride == 8
    assert all(o % 256 == 0 for o in offs)
    assert offs == sorted(offs) and len(set(offs)) == len(offs)
    assert list(L.slot_base)[2:5] == [0, 1024, 1280] and L.total_slots == 1408
    H, C, T = 4, 1024, 1408
    assert L.layer_stride[0] == H * (C // 64) * 9216            # base group records
    assert L.layer_stride[1] == H * (T // 64) * 9216            # residual group records
    assert L.layer_stride[5] == 4 * H * 64 * 128 * 2            # tail_k
    for i, name in enumerate(abi.ARRAY_NAMES[:-1]):
        nxt = getattr(L, abi.ARRAY_NAMES[i + 1])
        assert getattr(L, name) + 2 * L.layer_stride[i] == nxt
    assert L.total_bytes >= L.status + 64


@pytest.mark.parametrize("kw,st", [
    (dict(capacity=1000), abi.FL_ERR_INVALID),
    (dict(loops=33), abi.FL_ERR_INVALID),
    (dict(max_select=0), abi.FL_ERR_INVALID),
    (dict(res_capacity={2: 100}), abi.FL_ERR_INVALID),
])
def test_bad_dims_are_rejected(kw, st):
    out = abi.fl_layout()
    assert abi._c_cache_layout(ctypes.byref(_dims(**kw)), ctypes.byref(out)) == st


def test_unsupported_head_dim_and_group():
    d = _dims()
    d.head_dim = 64
    assert abi._c_cache_layout(ctypes.byref(d), ctypes.byref(abi.fl_layout())) == abi.FL_ERR_UNSUPPORTED
    d = _dims()
    d.group = 32
    assert abi._c_workspace_bytes(ctypes.byref(d)) == 0


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below fails validation first


def test_reader_arguments_are_validated_before_launch():
    d = _dims()
    ws = abi.fl_workspace_bytes(d)
    dense = lambda **k: abi._c_dense(ctypes.byref(d), k.get("cache", FAKE), k.get("layer", 0), k.get("loop", 1),
                                     k.get("n_q", 64), k.get("n_tail", 1), FAKE, k.get("kn"), k.get("vn"), FAKE,
                                     1, FAKE, k.get("ws", ws), None)
    assert dense(cache=None) == abi.FL_ERR_INVALID
    assert dense(layer=2) == abi.FL_ERR_INVALID
    assert dense(loop=5) == abi.FL_ERR_INVALID
    assert dense(loop=0) == abi.FL_ERR_INVALID
    assert dense(n_q=65) == abi.FL_ERR_INVALID
    assert dense(n_tail=0) == abi.FL_ERR_INVALID
    assert dense(n_tail=65) == abi.FL_ERR_INVALID
    assert dense(n_q=1024) == abi.FL_ERR_INVALID          # exceeds capacity
    assert dense(kn=FAKE) == abi.FL_ERR_INVALID            # k_new without v_new
    assert dense(ws=ws - 1) == abi.FL_ERR_WORKSPACE
    sparse = lambda k_sel, prev=FAKE: abi._c_sparse(ctypes.byref(d), FAKE, 0, 3, 64, 1, k_sel, FAKE, None, None,
                                                    prev, FAKE, FAKE, ws, None)
    assert sparse(0) == abi.FL_ERR_INVALID
    assert sparse(66) == abi.FL_ERR_INVALID               # more than N
    assert sparse(10, prev=None) == abi.FL_ERR_INVALID    # o_prev is required
    sel = lambda **k: abi._c_select(ctypes.byref(d), FAKE, k.get("l0", 0), k.get("nl", 1), k.get("loop", 3),
                                    k.get("n_q", 64), 1, k.get("k_sel", 10), None)
    assert sel(nl=3) == abi.FL_ERR_INVALID
    assert sel(loop=1) == abi.FL_ERR_INVALID              # a selection prepares a sparse loop >= 2
    assert sel(k_sel=129) == abi.FL_ERR_INVALID           # above max_select
    step = lambda **k: abi._c_step(ctypes.byref(d), FAKE, 64, 1, k.get("dl", 2), k.get("k_sel", 10),
                                   k.get("lf", 1), k.get("ll", 4), FAKE, None, None, FAKE, FAKE, ws, None, None)
    assert step(dl=5) == abi.FL_ERR_INVALID
    assert step(lf=3, ll=2) == abi.FL_ERR_INVALID
    assert step(ll=5) == abi.FL_ERR_INVALID
    assert step(k_sel=0) == abi.FL_ERR_INVALID
    assert step(dl=0, lf=1) == abi.FL_ERR_INVALID         # first loop cannot be sparse
    big = _dims(capacity=385024 + 128, max_select=10)
    assert abi._c_select(ctypes.byref(big), FAKE, 0, 1, 3, 385024, 1, 10, None) == abi.FL_ERR_UNSUPPORTED
    # the host-buffer step validates the whole step (the same rules) before any copy is enqueued
    step_io = lambda **k: abi._c_step_io(ctypes.byref(d), FAKE, 64, 1, k.get("dl", 2), k.get("k_sel", 10),
                                         k.get("lf", 1), k.get("ll", 4), k.get("qkv", FAKE), k.get("hq", FAKE),
                                         FAKE, k.get("ho", FAKE), FAKE, ws, None, None, None)
    assert step_io(dl=5) == abi.FL_ERR_INVALID
    assert step_io(lf=3, ll=2) == abi.FL_ERR_INVALID
    assert step_io(k_sel=0) == abi.FL_ERR_INVALID
    assert step_io(dl=0, lf=1) == abi.FL_ERR_INVALID
    assert step_io(qkv=None) == abi.FL_ERR_INVALID
    assert step_io(hq=None) == abi.FL_ERR_INVALID
    assert step_io(ho=None) == abi.FL_ERR_INVALID


def test_encoder_arguments_are_validated_before_launch():
    d = _dims()
    base = lambda row0, n: abi._c_encode_base(ctypes.byref(d), FAKE, 0, row0, n, FAKE, FAKE, 128 * 64, None)
    assert base(32, 64) == abi.FL_ERR_INVALID
    assert base(0, 100) == abi.FL_ERR_INVALID
    assert base(1024, 64) == abi.FL_ERR_INVALID
    res = lambda **k: abi._c_encode_residual(ctypes.byref(d), FAKE, 0, k.get("loop", 3), 0, 256,
                                             k.get("slot0", 0), FAKE, k.get("n", 10), FAKE, FAKE,
                                             128 * 256, 0, None)
    assert res(loop=1) == abi.FL_ERR_INVALID
    assert res(slot0=32) == abi.FL_ERR_INVALID
    assert res(slot0=192, n=100) == abi.FL_ERR_INVALID    # beyond loop 3's 256 slots
    assert res(n=300) == abi.FL_ERR_INVALID               # more rows than the span
    tail = abi._c_write_tail(ctypes.byref(d), FAKE, 0, 1, 60, 8, FAKE, FAKE, 128 * 8, None)
    assert tail == abi.FL_ERR_INVALID


def test_status_strings():
    for st in (abi.FL_OK, abi.FL_ERR_INVALID, abi.FL_ERR_UNSUPPORTED, abi.FL_ERR_CUDA, abi.FL_ERR_WORKSPACE,
               abi.FL_ERR_DEVICE):
        assert abi.fl_status_string(st).startswith("FL_")


def test_host_bookkeeping_helpers():
    assert [round_up(x) for x in (0, 1, 64, 65, 8176)] == [0, 64, 64, 128, 8192]
    assert split_prefill(32768) == (32704, 64) and split_prefill(100) == (64, 36)


def test_noalloc_sparse_validation():
    """The no-workspace sparse entry point validates on the host like the workspace one
    and refuses a scratch larger than its static array (no compute: null cache)."""
    d = abi.Dims(layers=1, heads=4, loops=4, capacity=1024, res_capacity={2: 1024, 3: 256, 4: 128}, max_select=128)
    code = abi._c_sparse_noalloc(ctypes.byref(d), None, 0, 3, 960, 1, 10, None, None, None, None, None, None)
    assert code == abi.FL_ERR_INVALID
    # a scratch beyond the static array is refused before any CUDA call
    buf = ctypes.create_string_buffer(256)
    p = (ctypes.addressof(buf) + 15) // 16 * 16
    big = abi.Dims(layers=1, heads=1100, loops=4, capacity=1024, res_capacity={2: 1024, 3: 256, 4: 128},
                   max_select=128)
    code = abi._c_sparse_noalloc(ctypes.byref(big), p, 0, 3, 960, 1, 10, p, None, None, p, p, None)
    assert code == abi.FL_ERR_UNSUPPORTED


def test_int2_records_take_5120_bytes_and_codecs_are_checked():
    dims = dict(layers=2, heads=3, loops=4, capacity=1024, max_select=128, res_capacity={2: 1024, 3: 512, 4: 256})
    L4 = abi.fl_cache_layout(abi.Dims(**dims))
    L2 = abi.fl_cache_layout(abi.Dims(**dims, codec=abi.FL_CODEC_RESIDUAL_INT2))
    T = 1024 + 512 + 256
    assert L4.total_slots == L2.total_slots == T
    rrec = abi.ARRAY_NAMES.index("rrec")
    assert L4.layer_stride[rrec] == 3 * (T // 64) * 9216
    assert L2.layer_stride[rrec] == 3 * (T // 64) * 5120
    assert L2.total_bytes < L4.total_bytes
    bad = abi.Dims(**dims, codec=3)
    with pytest.raises(abi.FlashLoopError) as e:
        abi.fl_cache_layout(bad)
    assert e.value.status == abi.FL_ERR_UNSUPPORTED


def test_fused_flush_plans_are_validated_before_launch():
    """fl_decode_step_flush refuses the codec variants (the fused flush writes 4-bit
    residual stores only) and plans whose active sets do not nest or whose slots are not
    64-aligned, before any launch."""
    good = [0, 0, 0b111, 0b011, 0b001]
    slots = [[0, 0, 64, 0, 0], [0, 0, 128, 0, 0]]          # two layers
    for codec, plan, st in [
        (abi.FL_CODEC_FULL_INT4, abi.Flush(good, slots), abi.FL_ERR_UNSUPPORTED),
        (abi.FL_CODEC_RESIDUAL_INT2, abi.Flush(good, slots), abi.FL_ERR_UNSUPPORTED),
        (abi.FL_CODEC_RESIDUAL_INT4, abi.Flush([0, 0, 0b01, 0b11, 0], slots), abi.FL_ERR_INVALID),
        (abi.FL_CODEC_RESIDUAL_INT4, abi.Flush(good, [[0, 0, 32, 0, 0]] * 2), abi.FL_ERR_INVALID),
        (abi.FL_CODEC_RESIDUAL_INT4, abi.Flush(good, [[0, 0, 1024, 0, 0]] * 2), abi.FL_ERR_INVALID),
    ]:
        d = _dims(codec=codec)
        ws = abi.fl_workspace_bytes(d)
        got = abi._c_step_flush(ctypes.byref(d), FAKE, 64, 64, 2, 10, 1, 4, FAKE, None, None, FAKE, FAKE, ws,
                                None, ctypes.byref(plan), None)
        assert got == st, (codec, got)


@pytest.mark.parametrize("loops", [4, 8, 9, 32])
def test_sparse_split_counts_fit_the_plan_copy_and_the_workspace(loops):
    """For every k_sel the sparse reader accepts, its split count leaves each CTA a share
    of the gather plan that fits the CTA's 1024-word shared-memory copy, and the workspace
    of fl_workspace_bytes holds that many partials per head -- including the deep 32-loop
    cache with every column selected (K_sel = N = 8192, 36-word plan entries), where 256
    splits would not do."""
    cap = 8192 + 128
    d = abi.Dims(layers=1, heads=16, loops=loops, capacity=cap, max_select=cap,
                 res_capacity={r: cap for r in range(2, loops + 1)})
    L = abi.fl_cache_layout(d)
    base_ws = abi.fl_workspace_bytes(d)
    for sms in (1, 148, 160, 1024):
        for loop in sorted({2, 3, min(8, loops), loops}):
            # the loop <= 8 reader of the method's codec copies 2048 plan words per CTA, the
            # loop > 8 reader 1024
            per_cta = (2048 if loop <= 8 else 1024) // L.plan_stride
            for k_sel in (1, 7, 31, 820, 3277, 7168, 7169, 8192, cap):
                n, capacity = abi.fl_sparse_splits(d, loop, k_sel, sms)
                assert 1 <= n <= capacity, (sms, loop, k_sel, n, capacity)
                assert -(-k_sel // n) <= per_cta, (sms, loop, k_sel, n)
                # the workspace holds `capacity` partials of 260 floats per head, then the tickets
                assert base_ws >= 16 * capacity * 260 * 4 + 16 * 4
    if loops == 32:
        n, capacity = abi.fl_sparse_splits(d, 32, 8192, 148)
        assert n > 256 and capacity >= n
    # the codec variants read through the loop <= 8 reader of 1024 plan words
    dv = abi.Dims(layers=1, heads=16, loops=loops, capacity=cap, max_select=cap,
                  res_capacity={r: cap for r in range(2, loops + 1)}, codec=abi.FL_CODEC_FULL_INT4)
    for k_sel in (820, 8192):
        n, capacity = abi.fl_sparse_splits(dv, 3, k_sel, 148)
        assert -(-k_sel // n) <= 1024 // L.plan_stride and n <= capacity
    with pytest.raises(abi.FlashLoopError):
        abi.fl_sparse_splits(d, 1, 10, 148)          # loop 1 is never sparse
    with pytest.raises(abi.FlashLoopError):
        abi.fl_sparse_splits(d, 2, cap + 1, 148)     # above max_select

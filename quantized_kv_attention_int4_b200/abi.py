"""ctypes binding of libflashloop_b200.so: the C ABI of include/flashloop.h, same names.

Argument marshalling only: every wrapper checks tensor placement, dtype and
contiguity, passes raw device pointers and the current CUDA stream, and raises
FlashLoopError on a non-OK status.  All compute runs in the library's kernels.
Importing this module without the built library raises ImportError.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

LIB_PATH = _build.LIB_PATH
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing; build it with `python -m quantized_kv_attention_int4_b200.build`")
lib = ctypes.CDLL(LIB_PATH)

MAX_LOOPS = 32
HEAD_DIM = 128
GROUP = 64
TAIL = 64
MAX_SELECT_COLS = 385024
N_ARRAYS = 14
ARRAY_NAMES = ("brec", "rrec", "mask", "first", "depth", "tail_k", "tail_v", "score", "tag", "offset", "sel",
               "mass", "unsel", "plan")
GROUP_RECORD = 9216
GROUP_RECORD_INT2 = 5120
# codecs of the loop r >= 2 stores (fl_dims.codec)
FL_CODEC_RESIDUAL_INT4, FL_CODEC_FULL_INT4, FL_CODEC_RESIDUAL_INT2 = 0, 1, 2

FL_OK, FL_ERR_INVALID, FL_ERR_UNSUPPORTED, FL_ERR_CUDA, FL_ERR_WORKSPACE, FL_ERR_DEVICE = 0, -1, -2, -3, -4, -6
# device error codes recorded in status words (include/flashloop.h)
FL_DEV_ROWS_ORDER, FL_DEV_ROWS_RANGE, FL_DEV_NOT_NESTED, FL_DEV_SEL_RANGE, FL_DEV_TAG_RANGE, FL_DEV_TIMEOUT = 1, 2, 3, 4, 5, 6
EXPORTED = ("fl_version", "fl_status_string", "fl_cache_layout", "fl_cache_init", "fl_workspace_bytes",
            "fl_workspace_init", "fl_write_tail", "fl_encode_base", "fl_encode_residual",
            "fl_decode_attn_dense", "fl_select_topk", "fl_decode_attn_sparse", "fl_decode_step",
            "fl_read_status", "fl_decode_attn_sparse_noalloc", "fl_decode_step_flush", "fl_select_active",
            "fl_prefill_attn_sparse", "fl_sparse_splits", "fl_decode_step_io")


class fl_dims(ctypes.Structure):
    _fields_ = [("layers", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("group", ctypes.c_int32), ("loops", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("max_select", ctypes.c_int32), ("res_capacity", ctypes.c_int32 * (MAX_LOOPS + 1)),
                ("codec", ctypes.c_int32)]


class fl_layout(ctypes.Structure):
    _fields_ = ([("total_bytes", ctypes.c_uint64)]
                + [(n, ctypes.c_uint64) for n in ARRAY_NAMES]
                + [("status", ctypes.c_uint64), ("layer_stride", ctypes.c_uint64 * N_ARRAYS),
                   ("plan_stride", ctypes.c_int32), ("slot_base", ctypes.c_int32 * (MAX_LOOPS + 1)),
                   ("total_slots", ctypes.c_int32)])


class fl_flush(ctypes.Structure):
    _fields_ = [("active", ctypes.c_uint64 * (MAX_LOOPS + 1)), ("slot0", ctypes.POINTER(ctypes.c_int32))]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_L = ctypes.c_int64
_DP = ctypes.POINTER(fl_dims)


def _sig(name, res, *args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_c_version = _sig("fl_version", ctypes.c_char_p)
_c_status_string = _sig("fl_status_string", ctypes.c_char_p, _I)
_c_cache_layout = _sig("fl_cache_layout", _I, _DP, ctypes.POINTER(fl_layout))
_c_cache_init = _sig("fl_cache_init", _I, _DP, _P, _P)
_c_workspace_bytes = _sig("fl_workspace_bytes", ctypes.c_size_t, _DP)
_c_workspace_init = _sig("fl_workspace_init", _I, _DP, _P, ctypes.c_size_t, _P)
_c_write_tail = _sig("fl_write_tail", _I, _DP, _P, _I, _I, _I, _I, _P, _P, _L, _P)
_c_encode_base = _sig("fl_encode_base", _I, _DP, _P, _I, _I, _I, _P, _P, _L, _P)
_c_encode_residual = _sig("fl_encode_residual", _I, _DP, _P, _I, _I, _I, _I, _I, _P, _I, _P, _P, _L, _I, _P)
_c_dense = _sig("fl_decode_attn_dense", _I, _DP, _P, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P,
                ctypes.c_size_t, _P)
_c_select = _sig("fl_select_topk", _I, _DP, _P, _I, _I, _I, _I, _I, _I, _P)
_c_sparse = _sig("fl_decode_attn_sparse", _I, _DP, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                 ctypes.c_size_t, _P)
_c_sparse_noalloc = _sig("fl_decode_attn_sparse_noalloc", _I, _DP, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                         _P)
_c_step = _sig("fl_decode_step", _I, _DP, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, ctypes.c_size_t,
                ctypes.POINTER(ctypes.c_void_p), _P)
_c_step_flush = _sig("fl_decode_step_flush", _I, _DP, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                      ctypes.c_size_t, ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(fl_flush), _P)
_c_select_active = _sig("fl_select_active", _I, _P, _P, _I, _I, _L, _P, _I, _I, _P, _P, _P, _P)
_c_prefill = _sig("fl_prefill_attn_sparse", _I, _P, _P, _I, _P, _P, _I, _I, _L, _L, _P, _L, _P, _P)
_c_read_status = _sig("fl_read_status", _I, _DP, _P, ctypes.POINTER(ctypes.c_int32), _I, _P)
_c_step_io = _sig("fl_decode_step_io", _I, _DP, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, ctypes.c_size_t,
                   ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(fl_flush), _P)
_c_sparse_splits = _sig("fl_sparse_splits", _I, _DP, _I, _I, _I, ctypes.POINTER(ctypes.c_int32),
                        ctypes.POINTER(ctypes.c_int32))


class FlashLoopError(RuntimeError):
    def __init__(self, where: str, status: int):
        super().__init__(f"{where}: {fl_status_string(status)}")
        self.status = status


def _check(where: str, st: int):
    if st != FL_OK:
        raise FlashLoopError(where, st)


def Dims(layers: int, heads: int, loops: int, capacity: int, max_select: int, res_capacity,
         codec: int = FL_CODEC_RESIDUAL_INT4) -> fl_dims:
    """fl_dims with head_dim 128 / group 64; res_capacity[r] for r = 2..loops (mapping or list);
    codec: FL_CODEC_* of the loop r >= 2 stores (the method's 4-bit residuals by default)."""
    d = fl_dims()
    d.layers, d.heads, d.head_dim, d.group = layers, heads, HEAD_DIM, GROUP
    d.loops, d.capacity, d.max_select, d.codec = loops, capacity, max_select, codec
    items = res_capacity.items() if isinstance(res_capacity, dict) else enumerate(res_capacity)
    for r, v in items:
        d.res_capacity[r] = int(v)
    return d


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(t, dtype, name):
    """A host tensor's data pointer (pinned memory keeps the library's copies asynchronous)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if t.dtype != dtype or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous {dtype} host tensor")
    return ctypes.c_void_p(t.data_ptr())


def _rows_tensor(x, name):
    """BF16 [H][n][128] with a unit-stride last dimension; returns (ptr, head_stride)."""
    if x.dim() != 3 or x.shape[2] != HEAD_DIM or x.stride(2) != 1 or x.stride(1) != HEAD_DIM:
        raise ValueError(f"{name} must be [H][n][128] with contiguous rows")
    return _ptr(x, torch.bfloat16, name), x.stride(0)


# ---------------------------------------------------------------------------
def fl_version() -> str:
    return _c_version().decode()


def fl_status_string(st: int) -> str:
    return _c_status_string(int(st)).decode()


def fl_cache_layout(dims: fl_dims) -> fl_layout:
    out = fl_layout()
    _check("fl_cache_layout", _c_cache_layout(ctypes.byref(dims), ctypes.byref(out)))
    return out


def fl_cache_init(dims, cache, stream=None):
    _check("fl_cache_init", _c_cache_init(ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), _stream(stream)))


def fl_workspace_bytes(dims) -> int:
    return int(_c_workspace_bytes(ctypes.byref(dims)))


def fl_sparse_splits(dims: fl_dims, loop: int, k_sel: int, sm_count: int):
    """(splits, capacity): split-K partitions per head of the loop-`loop` sparse reader over
    k_sel columns on a device with sm_count SMs, and the partials per head a workspace holds."""
    n, cap = ctypes.c_int32(0), ctypes.c_int32(0)
    _check("fl_sparse_splits", _c_sparse_splits(ctypes.byref(dims), loop, k_sel, sm_count, ctypes.byref(n),
                                                ctypes.byref(cap)))
    return n.value, cap.value

def fl_workspace_init(dims, ws, stream=None):
    _check("fl_workspace_init", _c_workspace_init(ctypes.byref(dims), _ptr(ws, torch.uint8, "ws"),
                                                  ws.numel(), _stream(stream)))


def fl_write_tail(dims, cache, layer, loop, row0, k, v, stream=None):
    kp, ks = _rows_tensor(k, "k")
    vp, vs = _rows_tensor(v, "v")
    if ks != vs or k.shape != v.shape:
        raise ValueError("k and v must have the same shape and strides")
    _check("fl_write_tail", _c_write_tail(ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), layer, loop,
                                          row0, k.shape[1], kp, vp, ks, _stream(stream)))


def fl_encode_base(dims, cache, layer, row0, k, v, stream=None):
    kp, ks = _rows_tensor(k, "k")
    vp, vs = _rows_tensor(v, "v")
    if ks != vs or k.shape != v.shape:
        raise ValueError("k and v must have the same shape and strides")
    _check("fl_encode_base", _c_encode_base(ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), layer, row0,
                                            k.shape[1], kp, vp, ks, _stream(stream)))


def fl_encode_residual(dims, cache, layer, loop, row0, n_span, slot0, rows, k, v, compact, stream=None):
    n = 0 if rows is None else rows.numel()
    if n:
        kp, ks = _rows_tensor(k, "k")
        vp, vs = _rows_tensor(v, "v")
        if ks != vs or k.shape != v.shape:
            raise ValueError("k and v must have the same shape and strides")
        rp = _ptr(rows, torch.int32, "rows")
    else:
        kp = vp = rp = None
        ks = 0
    _check("fl_encode_residual", _c_encode_residual(ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), layer,
                                                    loop, row0, n_span, slot0, rp, n, kp, vp, ks,
                                                    1 if compact else 0, _stream(stream)))


def fl_decode_attn_dense(dims, cache, layer, loop, n_q, n_tail, q, k_new, v_new, o, keep_scores, ws, stream=None):
    _check("fl_decode_attn_dense", _c_dense(
        ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), layer, loop, n_q, n_tail,
        _ptr(q, torch.bfloat16, "q"), _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        _ptr(o, torch.float32, "o"), 1 if keep_scores else 0, _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream)))


def fl_select_topk(dims, cache, layer0, n_layers, loop, n_q, n_tail, k_sel, stream=None):
    _check("fl_select_topk", _c_select(ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), layer0, n_layers,
                                       loop, n_q, n_tail, k_sel, _stream(stream)))


def fl_decode_attn_sparse(dims, cache, layer, loop, n_q, n_tail, k_sel, q, k_new, v_new, o_prev, o, ws,
                          stream=None):
    _check("fl_decode_attn_sparse", _c_sparse(
        ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), layer, loop, n_q, n_tail, k_sel,
        _ptr(q, torch.bfloat16, "q"), _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        _ptr(o_prev, torch.float32, "o_prev"), _ptr(o, torch.float32, "o"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream)))


def fl_decode_attn_sparse_noalloc(dims, cache, layer, loop, n_q, n_tail, k_sel, q, k_new, v_new, o_prev, o,
                                  stream=None):
    """fl_decode_attn_sparse with the library's static scratch instead of a workspace."""
    _check("fl_decode_attn_sparse_noalloc", _c_sparse_noalloc(
        ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), layer, loop, n_q, n_tail, k_sel,
        _ptr(q, torch.bfloat16, "q"), _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        _ptr(o_prev, torch.float32, "o_prev"), _ptr(o, torch.float32, "o"), _stream(stream)))


def Flush(active, slot0) -> fl_flush:
    """fl_flush from active[r] (64-bit row masks, index = loop) and slot0[l][r] (host ints)."""
    f = fl_flush()
    for r, m in enumerate(active):
        f.active[r] = int(m)
    rows = [list(x) for x in slot0]
    arr = (ctypes.c_int32 * (len(rows) * (MAX_LOOPS + 1)))()
    for l, row in enumerate(rows):
        for r, v in enumerate(row):
            arr[l * (MAX_LOOPS + 1) + r] = int(v)
    f.slot0 = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))
    f._keep = arr  # the struct points into this array
    return f


def fl_decode_step(dims, cache, n_q, n_tail, dense_loops, k_sel, loop_first, loop_last, q, k_new, v_new, o, ws,
                   events=None, stream=None, flush=None):
    """One loop-major decode step over every layer; q/k_new/v_new BF16 and o fp32, all [R+1][L][H][128].

    ``events``: None or a list of 2R+1 torch.cuda.Event (enable_timing) recorded at segment boundaries.
    ``flush``: None, or an fl_flush (see Flush): the step also quantises its full 64-row tail
    (fl_decode_step_flush).
    """
    ev = None
    if events is not None:
        for e in events:
            e.record()  # materialise the underlying cudaEvent_t
        ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    for t, name in ((q, "q"), (k_new, "k_new"), (v_new, "v_new")):
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous [R+1][L][H][128]")
    if not o.is_contiguous():
        raise ValueError("o must be contiguous [R+1][L][H][128]")
    args = (ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), n_q, n_tail, dense_loops, k_sel, loop_first,
            loop_last, _ptr(q, torch.bfloat16, "q"), _ptr(k_new, torch.bfloat16, "k_new"),
            _ptr(v_new, torch.bfloat16, "v_new"), _ptr(o, torch.float32, "o"), _ptr(ws, torch.uint8, "ws"),
            ws.numel(), ev)
    if flush is None:
        _check("fl_decode_step", _c_step(*args, _stream(stream)))
    else:
        _check("fl_decode_step_flush", _c_step_flush(*args, ctypes.byref(flush), _stream(stream)))



def fl_decode_step_io(dims, cache, n_q, n_tail, dense_loops, k_sel, loop_first, loop_last, qkv, host_qkv, o,
                      host_o, ws, events=None, stream=None, flush=None):
    """fl_decode_step_flush fed from and returning to host memory in one call.

    qkv: device BF16 [3][R+1][L][H][128] (q, k_new, v_new); host_qkv: host BF16
    [3][n][L][H][128] with n = loop_last - loop_first + 1; o: device fp32 [R+1][L][H][128];
    host_o: host fp32 [n][L][H][128] (valid after the stream is synchronised)."""
    ev = None
    if events is not None:
        for e in events:
            e.record()
        ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    if not qkv.is_contiguous() or not o.is_contiguous():
        raise ValueError("qkv and o must be contiguous")
    _check("fl_decode_step_io", _c_step_io(
        ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), n_q, n_tail, dense_loops, k_sel, loop_first, loop_last,
        _ptr(qkv, torch.bfloat16, "qkv"), _host_ptr(host_qkv, torch.bfloat16, "host_qkv"), _ptr(o, torch.float32, "o"),
        _host_ptr(host_o, torch.float32, "host_o"), _ptr(ws, torch.uint8, "ws"), ws.numel(), ev,
        ctypes.byref(flush) if flush is not None else None, _stream(stream)))

def fl_select_active(h_prev, h_cur, rows, k, rows_out, keys, status=None, stream=None):
    """A_r from A_{r-1}: the k tokens of ``rows`` (int32, ascending) whose hidden state
    changed most between h_prev and h_cur (BF16 [n_tokens][d], unit-stride rows), written
    ascending to rows_out (int32 [>= k]); keys (fp64 [>= len(rows)]) receives every
    candidate's squared relative change."""
    for t, name in ((h_prev, "h_prev"), (h_cur, "h_cur")):
        if t.dim() != 2 or t.stride(1) != 1:
            raise ValueError(f"{name} must be [n_tokens][d] with unit-stride rows")
    if h_prev.shape != h_cur.shape or h_prev.stride() != h_cur.stride():
        raise ValueError("h_prev and h_cur must have the same shape and strides")
    n = rows.numel()
    if keys.numel() < n or (k > 0 and rows_out.numel() < k):
        raise ValueError("keys must hold len(rows) entries and rows_out k entries")
    _check("fl_select_active", _c_select_active(
        _ptr(h_prev, torch.bfloat16, "h_prev"), _ptr(h_cur, torch.bfloat16, "h_cur"), h_prev.shape[0],
        h_prev.shape[1], h_prev.stride(0), _ptr(rows, torch.int32, "rows"), n, k,
        _ptr(rows_out, torch.int32, "rows_out"), _ptr(keys, torch.float64, "keys"),
        _ptr(status, torch.int32, "status"), _stream(stream)))


def fl_prefill_attn_sparse(q, pos, k, v, o, status=None, stream=None):
    """Causal attention of the active tokens: q BF16 [H][n_act][128] (compact), pos int32
    [n_act] (ascending token positions), k, v BF16 [H][N][128], o fp32 [H][n_act][128]."""
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        if t.dim() != 3 or t.shape[2] != HEAD_DIM or t.stride(2) != 1 or t.stride(1) != HEAD_DIM:
            raise ValueError(f"{name} must be [H][n][128] with contiguous rows")
    H, n_act = q.shape[0], q.shape[1]
    if k.shape != v.shape or k.stride() != v.stride() or k.shape[0] != H or o.shape[:2] != q.shape[:2]:
        raise ValueError("q, k, v, o shapes do not agree")
    if pos.numel() != n_act:
        raise ValueError("pos must hold one position per query row")
    _check("fl_prefill_attn_sparse", _c_prefill(
        _ptr(q, torch.bfloat16, "q"), _ptr(pos, torch.int32, "pos"), n_act, _ptr(k, torch.bfloat16, "k"),
        _ptr(v, torch.bfloat16, "v"), k.shape[1], H, q.stride(0), k.stride(0), _ptr(o, torch.float32, "o"),
        o.stride(0), _ptr(status, torch.int32, "status"), _stream(stream)))


def fl_read_status(dims, cache, clear=True, stream=None):
    """(status, [first error code, detail, count]); synchronises the stream."""
    out = (ctypes.c_int32 * 3)()
    st = _c_read_status(ctypes.byref(dims), _ptr(cache, torch.uint8, "cache"), out, 1 if clear else 0,
                        _stream(stream))
    if st not in (FL_OK, FL_ERR_DEVICE):
        raise FlashLoopError("fl_read_status", st)
    return st, [out[0], out[1], out[2]]

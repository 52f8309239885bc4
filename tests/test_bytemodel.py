"""The byte model reproduces the storage figures the flozi guide prints.

Fixture: tests/golden/pages_storage_figures.json (flozi.net guide "FlashLoop:
store changes between repeated passes", section 1 Cell 1 and section 3 storage cell).
"""
import json
import os

from quantized_kv_attention_int4_b200 import bytemodel as bm

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_storage_figures.json")))


def test_bytes_per_token_loop_and_cache_size():
    per = bm.bf16_bytes_per_token_loop(G["layers"], G["heads"], G["head_dim"])
    assert per == G["bytes_per_token_loop"]
    tot = bm.bf16_cache_bytes(G["layers"], G["heads"], G["context"], G["loops"], G["head_dim"])
    assert tot == G["bf16_cache_gib"] * bm.GIB


def test_ideal_payload_tail_and_reduction():
    tot = G["bf16_cache_gib"] * bm.GIB
    pay = bm.ideal_int4_payload(tot, G["loops"], G["retained"]) / bm.GIB
    tail = bm.bf16_tail_extra(tot, G["context"], G["tail_tokens"]) / bm.GIB
    assert round(pay, 2) == G["ideal_int4_payload_gib"]
    assert round(tail, 2) == G["tail_extra_gib"]
    assert round(pay + tail, 2) == G["ideal_total_gib"]
    assert round(G["bf16_cache_gib"] / (pay + tail), 2) == G["ideal_reduction"]


def test_row_cost_is_144_bytes():
    assert bm.ROW_BYTES == 144 and bm.TAIL_ROW == 512


def test_sparse_bytes_counted_from_a_gather_plan():
    """bench.py's per-codec count of a sparse launch's rows, key groups and value-only
    rows, on a hand-made plan (one head: a base-only column, a column with stores 1..3
    and tag 2, a tail column)."""
    import types

    import numpy as np
    import torch

    import bench
    from quantized_kv_attention_int4_b200 import abi

    ms, ps, k, n_q = 4, 8, 3, 128
    plan = np.zeros((1, ms, ps), np.int32)
    plan[0, 0, :2] = [5, 1 | (1 << 8)]               # base only, tag 1
    plan[0, 1, :2] = [70, 2 | (3 << 8)]              # stores 1..3, tag 2
    plan[0, 1, 3:5] = [10, 70]                       # global slots in stores 2 and 3
    plan[0, 2, :2] = [130, 2]                        # a tail column
    raw = torch.from_numpy(plan.view(np.uint8).reshape(-1).copy())

    def cache(codec):
        return types.SimpleNamespace(H=1, n_q=n_q, codec=codec, dims=types.SimpleNamespace(max_select=ms),
                                     layout=types.SimpleNamespace(plan_stride=ps), raw=lambda name, layer: raw)

    # residual codecs: rows 1 + 3, key groups: base blocks {0, 1} + slot groups {0} and {1}
    assert bench.sparse_bytes_from_plan(cache(abi.FL_CODEC_RESIDUAL_INT4), 1, k) == \
        bm.sparse_bytes(1, 2, 2, 4, 1, bm.CODE_ROW, 0)
    assert bench.sparse_bytes_from_plan(cache(abi.FL_CODEC_RESIDUAL_INT2), 1, k) == \
        bm.sparse_bytes(1, 2, 2, 4, 1, bm.CODE_ROW2, 0)
    # full state: one row per column (base block 0; store 3 slot group 1) and the value half
    # of store min(tag, stores) = 2 for the second column
    assert bench.sparse_bytes_from_plan(cache(abi.FL_CODEC_FULL_INT4), 1, k) == \
        bm.sparse_bytes(1, 2, 0, 2, 1, bm.CODE_ROW, 1)

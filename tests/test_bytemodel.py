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

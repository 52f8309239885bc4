"""Byte accounting for the FlashLoop cross-loop cache and its decode kernels.

Two parts:

* the storage arithmetic the flozi guide "FlashLoop: store changes between
  repeated passes" prints (section 1, Cell 1: bytes per (token, loop) of a BF16
  cross-loop cache; section 3: ideal INT4 payload with a 64-token BF16 tail),
  restated here so the figures can be checked;
* the algorithmic bytes of one launch of each decode kernel: what must cross
  HBM at least once, used as the numerator of achieved GB/s.

Per-token costs of the packed INT4 layout (head dim 128, group 64): 64 B of key
codes, 64 B of value codes, 8 B of value (scale, zero) and 8 B of key
(scale, zero) amortised over the 64 tokens of a key group: 144 B per stored
row, base or residual.  A BF16 tail row is 256 B of key plus 256 B of value.
"""
from __future__ import annotations

GIB = 1024 ** 3
HEAD_DIM = 128
GROUP = 64
CODE_ROW = HEAD_DIM // 2          # 64 B of packed 4-bit codes per row
VSZ_ROW = 8                       # two (scale, zero) fp16 pairs per value row
KSZ_GROUP = HEAD_DIM * 4          # (scale, zero) fp16 pair per channel per key group
ROW_BYTES = 2 * CODE_ROW + VSZ_ROW + KSZ_GROUP // GROUP   # 144
TAIL_ROW = 2 * HEAD_DIM * 2       # K + V in BF16
# a 2-bit residual row (FL_CODEC_RESIDUAL_INT2): 32 + 32 B of codes, the same scales
CODE_ROW2 = HEAD_DIM // 4
ROW_BYTES2 = 2 * CODE_ROW2 + VSZ_ROW + KSZ_GROUP // GROUP  # 80


def bf16_bytes_per_token_loop(layers: int, heads: int, head_dim: int = HEAD_DIM) -> int:
    """K and V of one token in one loop, all layers, BF16."""
    return layers * heads * head_dim * 2 * 2


def bf16_cache_bytes(layers: int, heads: int, context: int, loops: int, head_dim: int = HEAD_DIM) -> int:
    """A separate BF16 (K, V) per loop for every token."""
    return bf16_bytes_per_token_loop(layers, heads, head_dim) * context * loops


def ideal_int4_payload(bf16_total: float, loops: int, retained) -> float:
    """INT4 codes only (no scales): a quarter of each loop's BF16 share, times the rows kept."""
    return bf16_total / loops * (4 / 16) * sum(retained)


def bf16_tail_extra(bf16_total: float, context: int, tail: int = 64) -> float:
    """Extra bytes of keeping ``tail`` recent tokens in BF16 rather than INT4, every loop."""
    return bf16_total * (tail / context) * (1 - 4 / 16)


# ----------------------------------------------------------------------------
# Algorithmic bytes per launch (one layer, all heads)
# ----------------------------------------------------------------------------
def dense_bytes(heads: int, n_q: int, n_tail: int, res_rows: int, keep_scores: bool,
                res_row_bytes: int = ROW_BYTES) -> int:
    """One dense-reader launch of loop r.

    n_q quantised columns read their base rows, ``res_rows`` is the number of
    residual rows of loops 2..r that belong to those columns (``res_row_bytes``
    each), the tail rows are BF16.  Plus q (BF16), o (fp32), and with
    ``keep_scores`` the per-column log-score (fp32) and loop tag (u8) written for
    the selector.  With full-state stores every quantised column reads one row
    (its last store): pass res_rows = 0.
    """
    per_head = n_q * ROW_BYTES + res_rows * res_row_bytes + n_tail * TAIL_ROW + HEAD_DIM * 2 + HEAD_DIM * 4
    if keep_scores:
        per_head += (n_q + n_tail) * 5
    return heads * per_head


def sparse_bytes(heads: int, cols_quant: int, res_rows: int, key_groups: int, cols_tail: int,
                 res_code_row: int = CODE_ROW, value_rows: int = 0) -> int:
    """One sparse-reader launch, summed over heads.

    ``cols_quant``: selected quantised columns (over all heads); ``res_rows``:
    residual rows those columns carry up to this loop (``res_code_row`` bytes of
    key and of value codes each); ``key_groups``: distinct (store, key group)
    pairs the selected rows touch (512 B of key scales each); ``cols_tail``:
    selected tail columns; ``value_rows``: rows read for their value half only
    (full-state stores: a column's value at its tag loop when that is another
    store).  Each selected column also reads its index (4 B), writes its new
    log-score and loop tag (5 B); per head q, m, u and o are read or written.
    """
    row = 2 * CODE_ROW + VSZ_ROW
    cols = cols_quant + cols_tail
    return (cols_quant * row + res_rows * (2 * res_code_row + VSZ_ROW) + value_rows * (CODE_ROW + VSZ_ROW)
            + key_groups * KSZ_GROUP + cols_tail * TAIL_ROW
            + cols * (4 + 5) + heads * (HEAD_DIM * 2 + 4 + HEAD_DIM * 4 * 2))


def encode_base_bytes(heads: int, n_rows: int) -> int:
    """One base-encoder launch: BF16 keys and values in (512 B per row), the row's 144 B of
    codes and scales out."""
    return heads * n_rows * (TAIL_ROW + ROW_BYTES)


def encode_residual_bytes(heads: int, n_rows: int, loop: int, n_tokens: int, row_bytes: int = ROW_BYTES) -> int:
    """One residual-encoder launch of loop ``loop`` over ``n_rows`` active rows of a span of
    ``n_tokens``: each row's BF16 key and value in, the loop r-1 reconstruction it is taken
    against (the row's base row and its residual rows of loops 2..r-1, 144 B each), its new
    row out; plus the span's block metadata (mask 8 B, first slot 4 B per 64 tokens) and
    depth (1 B per row)."""
    return heads * n_rows * (TAIL_ROW + ROW_BYTES * (loop - 1) + row_bytes) + (n_tokens // GROUP) * 12 + n_rows

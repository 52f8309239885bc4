"""Host bookkeeping for a FlashLoop cross-loop cache held in one device buffer.

The C library is stateless: every call states the token range, slot offset and
column counts it works on.  This class keeps those numbers for a stack of layers
that advance through the same token timeline:

* ``n_q`` quantised tokens (a multiple of 64) and ``n_tail`` BF16 tail rows (1..64);
* per layer and loop, how many residual slots are used (each encode call starts a
  new 64-slot key group, so the next call begins at the next multiple of 64);
* the last loop each tail token is active in, which decides the rows of every
  residual store when the tail is flushed into INT4 (flashloop 0.1.0 PyPI
  description, "Configuration and supported scope": 64-token BF16 tail; FlashLoop
  project page, "The Method", Step 03: residuals for active tokens only).

``codec`` selects what the loop r >= 2 stores hold (``abi.FL_CODEC_*``): the method's
4-bit residuals, per-loop 4-bit full states, or 2-bit residuals.  The fused tail flush
(``step(..., flush=True)``) serves the first only; ``begin_token`` flushes any codec
through the encode entry points.

Every device operation goes through the ``abi`` wrappers.
"""
from __future__ import annotations

import torch

from . import abi

GROUP = 64
TAIL = 64


def round_up(x: int, m: int = GROUP) -> int:
    return (x + m - 1) // m * m


def split_prefill(n_cols: int) -> tuple[int, int]:
    """(n_q, n_tail) with n_q a multiple of 64 and 1 <= n_tail <= 64."""
    n_tail = n_cols - GROUP * ((n_cols - 1) // GROUP)
    return n_cols - n_tail, n_tail


class FlashLoopCache:
    def __init__(self, layers: int, heads: int, loops: int, capacity: int, res_capacity=None,
                 max_select: int | None = None, device="cuda", codec: int = abi.FL_CODEC_RESIDUAL_INT4):
        capacity = round_up(capacity)
        if res_capacity is None:
            res_capacity = {r: capacity for r in range(2, loops + 1)}
        if max_select is None:
            max_select = capacity
        self.L, self.H, self.R, self.capacity, self.codec = layers, heads, loops, capacity, codec
        self.device = torch.device(device)
        self.dims = abi.Dims(layers, heads, loops, capacity, max_select, res_capacity, codec)
        self.layout = abi.fl_cache_layout(self.dims)
        self.buf = torch.empty(self.layout.total_bytes, dtype=torch.uint8, device=self.device)
        abi.fl_cache_init(self.dims, self.buf)
        self.ws = torch.empty(abi.fl_workspace_bytes(self.dims), dtype=torch.uint8, device=self.device)
        abi.fl_workspace_init(self.dims, self.ws)
        self.n_q = 0
        self.n_tail = 0
        self.n_slots = [[0] * (loops + 1) for _ in range(layers)]
        self.n_rows = [[0] * (loops + 1) for _ in range(layers)]   # residual rows actually stored
        self.tail_depth: list[int] = []
        self._rows_cache: dict = {}
        self._plan = None   # (n_q, fl_flush) of a flushing step split over loop ranges

    # ---- views into the device buffer (for tests and inspection) -----------------
    def raw(self, name: str, layer: int) -> torch.Tensor:
        """The bytes of array ``name`` for one layer (uint8 view, no copy)."""
        i = abi.ARRAY_NAMES.index(name)
        off = getattr(self.layout, name) + self.layout.layer_stride[i] * layer
        return self.buf[off: off + self.layout.layer_stride[i]]

    def tail(self, which: str, layer: int, loop: int) -> torch.Tensor:
        """BF16 tail of one (layer, loop): [H][64][128] view."""
        n = self.H * TAIL * 128
        t = self.raw("tail_k" if which == "k" else "tail_v", layer)
        return t[(loop - 1) * n * 2: loop * n * 2].view(torch.bfloat16).view(self.H, TAIL, 128)

    @property
    def n_cols(self) -> int:
        return self.n_q + self.n_tail

    # ---- prefill -----------------------------------------------------------------
    def prefill_layer(self, layer: int, K: list, V: list, sets: list):
        """Encode one layer's prompt: K[r], V[r] BF16 [H][n][128] (r = 1..R), nested active sets.

        The last 1..64 prompt tokens stay in the BF16 tail of every loop.
        """
        n = K[1].shape[1]
        n_q, n_tail = split_prefill(n)
        d = self.dims
        if n_q:
            abi.fl_encode_base(d, self.buf, layer, 0, K[1][:, :n_q], V[1][:, :n_q])
        for r in range(2, self.R + 1):
            rows = sets[r][sets[r] < n_q].to(device=self.device, dtype=torch.int32)
            slot0 = round_up(self.n_slots[layer][r])
            abi.fl_encode_residual(d, self.buf, layer, r, 0, n_q, slot0, rows,
                                   K[r][:, :n_q], V[r][:, :n_q], compact=False)
            self.n_slots[layer][r] = slot0 + rows.numel()
            self.n_rows[layer][r] += rows.numel()
        for r in range(1, self.R + 1):
            abi.fl_write_tail(d, self.buf, layer, r, 0, K[r][:, n_q:], V[r][:, n_q:])
        depth = torch.zeros(n, dtype=torch.int64)
        for r in range(1, self.R + 1):
            depth[sets[r]] = r
        return n_q, n_tail, depth[n_q:].tolist()

    def set_timeline(self, n_q: int, n_tail: int, tail_depth):
        self.n_q, self.n_tail = n_q, n_tail
        self.tail_depth = list(tail_depth)

    # ---- decode --------------------------------------------------------------------
    def _flush_rows(self, r: int) -> torch.Tensor:
        key = (self.n_q, r, tuple(self.tail_depth))
        rows = self._rows_cache.get(key)
        if rows is None:
            idx = [self.n_q + i for i, dep in enumerate(self.tail_depth) if dep >= r]
            rows = torch.tensor(idx, dtype=torch.int32).to(self.device)
            self._rows_cache = {key: rows} if len(self._rows_cache) > 64 else {**self._rows_cache, key: rows}
        return rows

    def flush_layer(self, layer: int):
        """Encode the 64 tail rows of one layer into the base and residual stores."""
        assert self.n_tail == TAIL
        d = self.dims
        abi.fl_encode_base(d, self.buf, layer, self.n_q, self.tail("k", layer, 1), self.tail("v", layer, 1))
        for r in range(2, self.R + 1):
            rows = self._flush_rows(r)
            slot0 = round_up(self.n_slots[layer][r])
            abi.fl_encode_residual(d, self.buf, layer, r, self.n_q, TAIL, slot0, rows,
                                   self.tail("k", layer, r), self.tail("v", layer, r), compact=False)
            self.n_slots[layer][r] = slot0 + rows.numel()
            self.n_rows[layer][r] += rows.numel()

    def flush_plan(self):
        """The fl_flush that moves the current full tail into the INT4 stores inside a step.

        Loop r's residual store takes the tail rows whose last active loop is >= r, at the
        next 64-aligned slot of each layer's store (the slots fl_encode_residual would use).
        """
        assert self.n_tail == TAIL
        active = [0] * (self.R + 1)
        for r in range(2, self.R + 1):
            active[r] = sum(1 << i for i, dep in enumerate(self.tail_depth) if dep >= r)
        slot0 = [[0] + [0] + [round_up(self.n_slots[layer][r]) for r in range(2, self.R + 1)]
                 for layer in range(self.L)]
        return abi.Flush(active, slot0)

    def _flushed(self, plan):
        """Host bookkeeping once a step has written every store of the flushed tail."""
        for layer in range(self.L):
            for r in range(2, self.R + 1):
                n = bin(plan.active[r]).count("1")
                self.n_slots[layer][r] = plan.slot0[layer * (abi.MAX_LOOPS + 1) + r] + n
                self.n_rows[layer][r] += n
        self.n_q += TAIL
        self.n_tail = 0
        self.tail_depth = []

    def begin_token(self, layers=None):
        """Make room for the next token: flush a full tail (every layer), then add one row.

        A step run with ``flush=True`` has already moved its full tail into the INT4
        stores; otherwise the tail is flushed here with the encode entry points.
        The new row's per-loop key/value are written by the readers (k_new / v_new).
        """
        if self.n_tail == TAIL:
            for layer in (range(self.L) if layers is None else layers):
                self.flush_layer(layer)
            self.n_q += TAIL
            self.n_tail = 0
            self.tail_depth = []
        self.n_tail += 1
        self.tail_depth.append(self.R)

    # ---- readers -------------------------------------------------------------------
    def dense(self, layer, loop, q, o, k_new=None, v_new=None, keep_scores=True, stream=None):
        abi.fl_decode_attn_dense(self.dims, self.buf, layer, loop, self.n_q, self.n_tail, q, k_new, v_new, o,
                                 keep_scores, self.ws, stream)

    def select(self, layer0, n_layers, loop, k_sel, stream=None):
        abi.fl_select_topk(self.dims, self.buf, layer0, n_layers, loop, self.n_q, self.n_tail, k_sel, stream)

    def sparse(self, layer, loop, k_sel, q, o_prev, o, k_new=None, v_new=None, stream=None):
        abi.fl_decode_attn_sparse(self.dims, self.buf, layer, loop, self.n_q, self.n_tail, k_sel, q, k_new, v_new,
                                  o_prev, o, self.ws, stream)

    def step(self, dense_loops, k_sel, q, o, k_new=None, v_new=None, loop_first=1, loop_last=None, events=None,
             stream=None, flush=False):
        """Loops loop_first..loop_last of one decode step for every layer (native executor).

        With ``flush`` (the tail must hold 64 rows) each reader also quantises its loop's
        store of the tail group; once loop R has run, the tail is part of the INT4 cache.
        A step split over loop ranges keeps one plan for all of its calls.
        """
        loop_last = loop_last or self.R
        plan = None
        if flush:
            if self._plan is None or self._plan[0] != self.n_q:
                self._plan = (self.n_q, self.flush_plan())
            plan = self._plan[1]
        abi.fl_decode_step(self.dims, self.buf, self.n_q, self.n_tail, dense_loops, k_sel, loop_first,
                           loop_last, q, k_new, v_new, o, self.ws, events, stream, flush=plan)
        if plan is not None and loop_last == self.R:
            self._plan = None
            self._flushed(plan)

    def step_io(self, dense_loops, k_sel, qkv, host_qkv, o, host_o, loop_first=1, loop_last=None, events=None,
                stream=None, flush=False):
        """``step`` fed from and returning to host memory (fl_decode_step_io): the loops'
        q / k_new / v_new come from ``host_qkv`` (BF16 [3][n][L][H][128], pinned) into the
        device array ``qkv`` ([3][R+1][L][H][128]) and their outputs go from ``o`` to
        ``host_o`` ([n][L][H][128]), n = loop_last - loop_first + 1, in one call."""
        loop_last = loop_last or self.R
        plan = None
        if flush:
            if self._plan is None or self._plan[0] != self.n_q:
                self._plan = (self.n_q, self.flush_plan())
            plan = self._plan[1]
        abi.fl_decode_step_io(self.dims, self.buf, self.n_q, self.n_tail, dense_loops, k_sel, loop_first, loop_last,
                              qkv, host_qkv, o, host_o, self.ws, events, stream, flush=plan)
        if plan is not None and loop_last == self.R:
            self._plan = None
            self._flushed(plan)

    def status(self, clear=True):
        return abi.fl_read_status(self.dims, self.buf, clear)

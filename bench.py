"""Benchmark of the FlashLoop decode hot path on B200 (one JSON line on rank 0).

Workload (default): a 48-layer x 16-head x head-dim-128 cross-loop cache at 32K
context with 4 loops (Ouro-2.6B-shaped), INT4 base + nested 25 % / 10 % residuals
+ BF16 tail, synthetic seeded data.  A *step* decodes one token through every
layer and loop in loop-major order (loop r runs all layers before loop r+1):

    append token -> loop 1 dense (48) -> loop 2 dense (48, keeps scores)
    -> select for loop 3 (all layers, one launch) -> loop 3 sparse (48)
    -> select for loop 4 (one launch) -> loop 4 sparse (48)

Metric: sparse loop-4 decode attention (the loop-4 selection launch plus the 48
loop-4 sparse-reader launches), microseconds per step.  Also reported: the whole
step, the per-kernel averages measured with CUDA events on the launch stream, the
achieved HBM bandwidth against the measured peak, the oracle on the host cores,
and the same metric end to end from pinned host buffers.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {flashloop,reference}]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from quantized_kv_attention_int4_b200 import bytemodel  # noqa: E402

METRIC = "sparse loop-4 decode attention µs/step at 32K ctx; achieved HBM GB/s vs peak"
UNIT = "us/step"
DEFAULT_WORKLOAD = "cache_l48_h16_n32768"
FALLBACK_HBM_GBS = 6650.0


def _kernel_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu record, or None when the
    kernel's sources changed since that capture (the counters no longer describe it)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "kernel_traffic.json")) as f:
            rec = json.load(f)[kernel]
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, "quantized_kv_attention_int4_b200", "csrc", src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        return int(rec["dram_read_bytes"]) + int(rec["dram_write_bytes"])
    except Exception:
        return None


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# the GPU path
# ----------------------------------------------------------------------------
def replica_workload(w: synth.Workload, rank: int) -> synth.Workload:
    """Rank `rank`'s independent replica of the workload (weak scaling: same shapes,
    its own seeds, no data shared between ranks)."""
    return synth.Workload(**{**w.__dict__, "seed": w.seed + 100003 * rank})


def max_over_ranks(values, device):
    """Element-wise maximum of `values` over all ranks (the job's time is its slowest rank)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized() and \
            torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def build_cache(w: synth.Workload, layers: int, rank: int, device, new_tokens: int = 256, codec: int = 0):
    from quantized_kv_attention_int4_b200.cache import FlashLoopCache, round_up

    n = w.n_ctx
    sets = synth.active_sets(w, n)
    extra = (new_tokens + 63) // 64 * 64 + 64  # room for the decoded tokens and one tail
    cap = round_up(n + extra)
    res_cap = {r: round_up(min(cap, int((sets[r] < n).sum()) + extra + 64 * 4)) for r in range(2, w.loops + 1)}
    cache = FlashLoopCache(layers, w.heads, w.loops, cap, res_capacity=res_cap,
                           max_select=w.k_sel(cap), device=device, codec=codec)
    wr = replica_workload(w, rank)
    info = None
    for layer in range(layers):
        d = synth.prefill_layer(wr, layer, device=device, sets=sets)
        info = cache.prefill_layer(layer, d["K"], d["V"], sets)
        del d
    n_q, n_tail, tail_depth = info
    cache.set_timeline(n_q, n_tail, tail_depth)
    torch.cuda.synchronize()
    return cache, wr


def step_inputs(w: synth.Workload, layers: int, steps: int, device):
    """Per step: queries and the new token's k/v, BF16 [R+1][L][H][128] (slice 0 unused)."""
    out = []
    for s in range(steps):
        q = torch.stack([synth.queries(w, l, s + 1, device=device) for l in range(layers)], dim=1)
        toks = [synth.decode_token(w, l, s, device=device) for l in range(layers)]
        kn = torch.stack([torch.stack([torch.zeros_like(t["k"][1])] + t["k"][1:]) for t in toks], dim=1)
        vn = torch.stack([torch.stack([torch.zeros_like(t["v"][1])] + t["v"][1:]) for t in toks], dim=1)
        out.append((q.contiguous(), kn.contiguous(), vn.contiguous()))
    return out


class Step:
    """One decode step: append the token (host bookkeeping), then the native loop-major
    executor over every layer and loop.  The step in which the tail reaches 64 rows also
    quantises it inside its readers (fused flush); only a prompt that ends with a full tail
    is flushed by the encode launches, at the first token."""

    def __init__(self, cache, w, layers, device):
        self.c, self.w, self.L = cache, w, layers
        self.O = torch.zeros(w.loops + 1, layers, w.heads, 128, dtype=torch.float32, device=device)

    def launches(self, flushed: bool) -> int:
        """Kernels the native executor launches for one step: per dense loop a reader per
        layer; per sparse loop one selection for every layer, then for loops <= 8 (4-bit
        residual stores) one persistent reader for every layer and its combine, else a
        reader per layer.  Plus the encode launches of a first-token flush."""
        w, L = self.w, self.L
        n = 0
        for r in range(1, w.loops + 1):
            if r <= w.dense_loops:
                n += L
            elif r <= 8:
                n += 1 + 2
            else:
                n += 1 + L
        return n + (L * w.loops if flushed else 0)

    def run(self, q, kn, vn, ev=None, loop_first=1, loop_last=None):
        c, w = self.c, self.w
        if ev is not None:
            ev["start"].record()
        flushed = False
        if loop_first == 1:
            flushed = c.n_tail == 64
            c.begin_token()
        seg = [ev[k] for k in EXEC_EVENTS] if ev is not None else None
        c.step(w.dense_loops, w.k_sel(c.n_cols), q, self.O, kn, vn, loop_first=loop_first,
               loop_last=loop_last or w.loops, events=seg, flush=c.n_tail == 64)
        return self.launches(flushed)


EXEC_EVENTS = ("flushed", "sel1", "loop1", "sel2", "loop2", "select3", "loop3", "select4", "loop4")
SEGMENTS = ("start",) + EXEC_EVENTS


def sparse_bytes_from_state(cache, w, layers, loop, k_sel):
    """Algorithmic bytes of the loop-`loop` sparse readers, from the selections now in the cache."""
    H, n_q, N = cache.H, cache.n_q, cache.n_cols
    C = cache.capacity
    total = 0
    ms = cache.dims.max_select
    for l in range(layers):
        S = cache.raw("sel", l).view(torch.int32)[: H * ms].view(H, ms)[:, :k_sel].cpu().numpy()
        depth = cache.raw("depth", l)[:C].cpu().numpy().astype(np.int64)
        mask = cache.raw("mask", l).view(torch.int64)[: (w.loops + 1) * (C // 64)].view(w.loops + 1, C // 64)
        first = cache.raw("first", l).view(torch.int32)[: (w.loops + 1) * (C // 64)].view(w.loops + 1, C // 64)
        mask = mask.cpu().numpy().view(np.uint64)
        first = first.cpu().numpy()
        quant = S[S < n_q]
        cols_tail = int((S >= n_q).sum())
        dep = np.minimum(depth[quant], loop)
        res_rows = int(np.maximum(dep - 1, 0).sum())
        groups = 0
        for h in range(H):
            s = S[h][S[h] < n_q]
            groups += len(np.unique(s // 64))  # base key groups
            for rp in range(2, loop + 1):
                act = s[depth[s] >= rp]
                if act.size == 0:
                    continue
                b = act // 64
                t = (act % 64).astype(np.uint64)
                mk = mask[rp, b]
                low = mk & ((np.uint64(1) << t) - np.uint64(1))
                cnt = np.array([bin(int(x)).count("1") for x in low])
                gs = cache.layout.slot_base[rp] + first[rp, b] + cnt
                groups += len(np.unique(gs // 64))
        total += bytemodel.sparse_bytes(H, int(quant.size), res_rows, groups, cols_tail)
    return total / layers


def sparse_bytes_from_plan(cache, layers, k_sel):
    """Algorithmic bytes of one sparse-reader launch from the gather plans now in the cache,
    for the cache's codec: the rows, key groups and tag-loop value rows each selected
    column needs (the plan holds each column's tag, store count and residual slots)."""
    from quantized_kv_attention_int4_b200 import abi

    H, n_q, ms, ps = cache.H, cache.n_q, cache.dims.max_select, cache.layout.plan_stride
    full = cache.codec == abi.FL_CODEC_FULL_INT4
    total = 0
    for l in range(layers):
        plan = cache.raw("plan", l).view(torch.int32)[: H * ms * ps].view(H, ms, ps)[:, :k_sel].cpu().numpy()
        cols_quant = cols_tail = res_rows = value_rows = groups = 0
        for h in range(H):
            e = plan[h]
            j, st, lam = e[:, 0], (e[:, 1] >> 8) & 0xFF, e[:, 1] & 0xFF
            q = j < n_q
            cols_quant += int(q.sum())
            cols_tail += int((~q).sum())
            j, st, lam, e = j[q], st[q], lam[q], e[q]
            if full:
                # one row of store st (keys and values), and the value half of store min(tag, st)
                value_rows += int((np.minimum(lam, st) != st).sum())
                keys = set((j[st == 1] // 64).tolist())
                for s in range(2, int(st.max(initial=1)) + 1):
                    keys |= set((e[st == s, 1 + s].astype(np.int64) // 64 + (1 << 40)).tolist())
                groups += len(keys)
            else:
                res_rows += int(np.maximum(st - 1, 0).sum())
                groups += len(np.unique(j // 64))
                for s in range(2, int(st.max(initial=1)) + 1):
                    groups += len(np.unique(e[st >= s, 1 + s] // 64))
        code_row = bytemodel.CODE_ROW2 if cache.codec == abi.FL_CODEC_RESIDUAL_INT2 else bytemodel.CODE_ROW
        total += bytemodel.sparse_bytes(H, cols_quant, res_rows, groups, cols_tail, code_row, value_rows)
    return total / layers


def dense_bytes_avg(cache, w, layers, loop):
    H = cache.H
    tot = 0
    for l in range(layers):
        res_rows = sum(cache.n_rows[l][rp] for rp in range(2, loop + 1))
        tot += bytemodel.dense_bytes(H, cache.n_q, cache.n_tail, res_rows, keep_scores=(loop == w.dense_loops))
    return tot / layers


def run_gpu(args, rank, world):
    from quantized_kv_attention_int4_b200 import abi  # noqa: F401  (fails loudly without the library)

    device = torch.device("cuda", torch.cuda.current_device())
    w = synth.WORKLOADS[args.workload]
    layers = args.layers or w.layers
    t0 = time.time()
    cache, wr = build_cache(w, layers, rank, device, new_tokens=args.warmup + args.steps + args.e2e_steps)
    total_steps = args.warmup + args.steps
    inputs = step_inputs(wr, layers, total_steps + args.e2e_steps, device)
    step = Step(cache, wr, layers, device)
    setup_s = time.time() - t0

    for s in range(args.warmup):
        step.run(*inputs[s])
    torch.cuda.synchronize()
    st, info = cache.status()
    if st != 0:
        raise RuntimeError(f"device error during warm-up: {info}")

    evs = [{k: torch.cuda.Event(enable_timing=True) for k in SEGMENTS} for _ in range(args.steps)]
    sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                           else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[torch.cuda.current_device()]))
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    launches = 0
    for s in range(args.steps):
        launches += step.run(*inputs[args.warmup + s], ev=evs[s])
    t_end.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)

    seg = {k: [] for k in ("flush", "loop1", "loop2", "select3", "loop3", "select4", "loop4")}
    for e in evs:
        seg["flush"].append(e["start"].elapsed_time(e["flushed"]))
        seg["loop1"].append(e["flushed"].elapsed_time(e["loop1"]))
        seg["loop2"].append(e["loop1"].elapsed_time(e["loop2"]))
        seg["select3"].append(e["loop2"].elapsed_time(e["select3"]))
        seg["loop3"].append(e["select3"].elapsed_time(e["loop3"]))
        seg["select4"].append(e["loop3"].elapsed_time(e["select4"]))
        seg["loop4"].append(e["select4"].elapsed_time(e["loop4"]))
    mean = {k: float(np.mean(v)) for k, v in seg.items()}
    metric_us = (mean["select4"] + mean["loop4"]) * 1e3
    step_ms = total_ms / args.steps

    metric_us, step_ms, loop4_ms, dense_ms = max_over_ranks(
        [metric_us, step_ms, mean["loop4"], mean["loop1"] + mean["loop2"]], device)

    N = cache.n_cols
    k_sel = wr.k_sel(N)
    hbm, peak_kind = _peaks()
    sp_bytes = sparse_bytes_from_state(cache, wr, layers, 4, k_sel)
    sp_launch_us = loop4_ms * 1e3 / layers
    sp_gbs = sp_bytes / (sp_launch_us * 1e-6) / 1e9
    d_bytes = (dense_bytes_avg(cache, wr, layers, 1) + dense_bytes_avg(cache, wr, layers, 2)) / 2
    d_launch_us = dense_ms * 1e3 / (2 * layers)
    d_gbs = d_bytes / (d_launch_us * 1e-6) / 1e9

    e2e = run_e2e(step, cache, wr, layers, inputs[total_steps:], device) if args.e2e_steps else None
    del inputs, step, cache
    encode = run_encode(synth.WORKLOADS["layer_h16_n32768_decode256"], device, hbm) if args.encode else None
    deep = run_deep(device, hbm) if args.deep else None
    tokens = run_token_select(wr, device, hbm) if args.token_select else None
    codecs = run_codecs(w, device, hbm, layers=args.codec_layers) if args.codecs else None
    prefill = run_prefill(wr, device) if args.prefill else None
    return dict(metric_us=metric_us, step_ms=step_ms, seg=mean, clocks=clocks, launches=launches / args.steps,
                sp_bytes=sp_bytes, sp_launch_us=sp_launch_us, sp_gbs=sp_gbs, d_bytes=d_bytes,
                d_launch_us=d_launch_us, d_gbs=d_gbs, hbm=hbm, peak_kind=peak_kind, N=N, k_sel=k_sel,
                layers=layers, setup_s=setup_s, e2e=e2e, w=wr, tokens=tokens, prefill=prefill, codecs=codecs,
                encode=encode, deep=deep)


def run_codecs(w, device, hbm, layers=4, warmup=3, steps=5):
    """The codec variants of the loop r >= 2 stores (per-loop KIVI4 full state, INT2
    residuals; flozi guide, section 4) on the workload's per-layer sizes, `layers`
    layers: the step executor without tail flushes (the variants have none fused),
    CUDA events around the dense loops and the loop-4 selection and sparse loop.
    Both variants run on the staged readers, as the method does."""
    from quantized_kv_attention_int4_b200 import abi

    out = {}
    for codec, name in ((abi.FL_CODEC_FULL_INT4, "full_int4"), (abi.FL_CODEC_RESIDUAL_INT2, "residual_int2")):
        cache, wr = build_cache(w, layers, 0, device, new_tokens=warmup + steps, codec=codec)
        inputs = step_inputs(wr, layers, warmup + steps, device)
        O = torch.zeros(wr.loops + 1, layers, wr.heads, 128, dtype=torch.float32, device=device)
        evs = [{k: torch.cuda.Event(enable_timing=True) for k in EXEC_EVENTS} for _ in range(steps)]
        for s in range(warmup + steps):
            cache.begin_token()           # the prompt's full tail is flushed by the encoders at the first token
            seg = [evs[s - warmup][k] for k in EXEC_EVENTS] if s >= warmup else None
            q, kn, vn = inputs[s]
            cache.step(wr.dense_loops, wr.k_sel(cache.n_cols), q, O, kn, vn, events=seg)
        torch.cuda.synchronize()
        st, info = cache.status()
        if st != 0:
            raise RuntimeError(f"device error in the {name} codec measurement: {info}")
        ms = lambda a, b: float(np.mean([e[a].elapsed_time(e[b]) for e in evs]))
        dense_ms = ms("flushed", "loop2")
        sel_ms, sp_ms = ms("loop3", "select4"), ms("select4", "loop4")
        k_sel = wr.k_sel(cache.n_cols)
        sp_bytes = sparse_bytes_from_plan(cache, layers, k_sel)
        sp_us = sp_ms * 1e3 / layers
        d_bytes = 0.0
        for loop in (1, 2):
            for l in range(layers):
                if codec == abi.FL_CODEC_FULL_INT4:
                    rows, rb = 0, bytemodel.ROW_BYTES
                else:
                    rows, rb = sum(cache.n_rows[l][rp] for rp in range(2, loop + 1)), bytemodel.ROW_BYTES2
                d_bytes += bytemodel.dense_bytes(cache.H, cache.n_q, cache.n_tail, rows, loop == wr.dense_loops, rb)
        d_bytes /= 2 * layers
        d_us = dense_ms * 1e3 / (2 * layers)
        rrec = cache.layout.layer_stride[abi.ARRAY_NAMES.index("rrec")]
        out[name] = {
            "kernels": "dense_staged_kernel (loops 1-2), sparse_staged_kernel (loop 4)",
            "sparse_us_per_launch": sp_us, "sparse_bytes_per_launch": sp_bytes,
            "sparse_gbs": sp_bytes / (sp_us * 1e-6) / 1e9, "sparse_frac": sp_bytes / (sp_us * 1e-6) / 1e9 / hbm,
            "select4_us": sel_ms * 1e3,
            "dense_us_per_launch": d_us, "dense_bytes_per_launch": d_bytes,
            "dense_gbs": d_bytes / (d_us * 1e-6) / 1e9, "dense_frac": d_bytes / (d_us * 1e-6) / 1e9 / hbm,
            "residual_store_bytes_per_layer": int(rrec), "layers": layers, "steps": steps,
            "sparse_traffic": _kernel_traffic("sparse_staged_kernel_" + name),
            "dense_traffic": _kernel_traffic("dense_staged_kernel_" + name),
        }
        del cache, inputs, O
        torch.cuda.empty_cache()
    return out


def run_token_select(w, device, hbm, reps=5):
    """The token-sparse update selector (fl_select_active) on the workload's prompt with a
    hidden state of H x 128 = 2048 BF16 per token: the loop-3 ranking (A_3, 25 %, from
    every token) and the loop-4 ranking (A_4, 10 %, from A_3).  CUDA events on the launch
    stream, L2 flushed before each timed call; the change kernel alone is the k = 0 call
    (keys only), whose bytes are both hidden-state rows of every candidate."""
    from quantized_kv_attention_int4_b200 import abi
    from quantized_kv_attention_int4_b200.tokens import nested_active_sets

    n, d = w.n_ctx, w.heads * 128
    h = synth.hidden_states(w, n, d, device=device)
    sizes = [0] + [w.n_active(r, n) for r in range(1, w.loops + 1)]
    sets = nested_active_sets(h, sizes)
    keys = torch.empty(n, dtype=torch.float64, device=device)
    out3 = torch.empty(sizes[3], dtype=torch.int32, device=device)
    out4 = torch.empty(sizes[4], dtype=torch.int32, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    calls = {
        "change": lambda: abi.fl_select_active(h[1], h[2], sets[2], 0, None, keys),
        "a3": lambda: abi.fl_select_active(h[1], h[2], sets[2], sizes[3], out3, keys),
        "a4": lambda: abi.fl_select_active(h[2], h[3], out3, sizes[4], out4, keys),
    }
    times = {k: [] for k in calls}
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for rep in range(reps + 1):
        for name, fn in calls.items():
            flush.zero_()
            ev[0].record()
            fn()
            ev[1].record()
            torch.cuda.synchronize()
            if rep:
                times[name].append(ev[0].elapsed_time(ev[1]) * 1e3)
    assert torch.equal(out3, sets[3]) and torch.equal(out4, sets[4])
    t = {k: float(np.mean(v)) for k, v in times.items()}
    nbytes = n * d * 2 * 2 + n * (4 + 8)
    gbs = nbytes / (t["change"] * 1e-6) / 1e9
    del h, flush
    return {"bound": "hbm", "kernel": f"token_change_kernel (loop-3 ranking over {n} tokens x {d})",
            "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
            "traffic": _kernel_traffic("token_change_kernel"), "bytes_per_launch": nbytes,
            "us_per_launch": t["change"], "a3_us": t["a3"], "a4_us": t["a4"],
            "select_us_a3": t["a3"] - t["change"]}


def run_encode(w, device, hbm, reps=5):
    """The prefill encode of one 16-head layer of a 32K-token prompt (the layer that then
    decodes 256 tokens): the base encoder over every quantised token, then the
    residual encoder of loops 2..R over their active rows, each timed with CUDA events on the
    launch stream (a repetition re-encodes the same rows; inputs of 0.5 GB, larger than L2)."""
    from quantized_kv_attention_int4_b200 import abi
    from quantized_kv_attention_int4_b200.cache import FlashLoopCache, round_up, split_prefill

    n = w.n_ctx
    sets = synth.active_sets(w, n)
    d = synth.prefill_layer(w, 0, device=device, sets=sets)
    n_q, _ = split_prefill(n)
    cache = FlashLoopCache(1, w.heads, w.loops, round_up(n + 64), device=device)
    rows = {r: sets[r][sets[r] < n_q].to(device=device, dtype=torch.int32) for r in range(2, w.loops + 1)}
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(w.loops + 1)]
    times = {r: [] for r in range(1, w.loops + 1)}
    for rep in range(reps + 1):
        ev[0].record()
        abi.fl_encode_base(cache.dims, cache.buf, 0, 0, d["K"][1][:, :n_q], d["V"][1][:, :n_q])
        ev[1].record()
        for r in range(2, w.loops + 1):
            abi.fl_encode_residual(cache.dims, cache.buf, 0, r, 0, n_q, 0, rows[r], d["K"][r][:, :n_q],
                                   d["V"][r][:, :n_q], compact=False)
            ev[r].record()
        torch.cuda.synchronize()
        if rep:
            for r in range(1, w.loops + 1):
                times[r].append(ev[r - 1].elapsed_time(ev[r]) * 1e3)
    st, info = cache.status()
    if st != 0:
        raise RuntimeError(f"device error in the encode measurement: {info}")
    out = {}
    for r in range(1, w.loops + 1):
        us = float(np.mean(times[r]))
        if r == 1:
            nb, name = bytemodel.encode_base_bytes(w.heads, n_q), "encode_base_kernel"
        else:
            nb, name = bytemodel.encode_residual_bytes(w.heads, int(rows[r].numel()), r, n_q), "encode_residual_kernel"
        gbs = nb / (us * 1e-6) / 1e9
        out[f"loop{r}"] = {"kernel": name, "us_per_launch": us, "bytes_per_launch": nb, "achieved": gbs,
                           "frac": gbs / hbm, "rows": n_q if r == 1 else int(rows[r].numel())}
    tot_b = sum(v["bytes_per_launch"] for v in out.values())
    tot_us = sum(v["us_per_launch"] for v in out.values())
    del d, cache
    torch.cuda.empty_cache()
    return {"bound": "hbm", "kernel": "encode_base_kernel + encode_residual_kernel (loops 2..R)",
            "workload": f"one {w.heads}-head layer, {n_q} quantised tokens", "achieved": tot_b / (tot_us * 1e-6) / 1e9,
            "peak": hbm, "unit": "GB/s", "frac": tot_b / (tot_us * 1e-6) / 1e9 / hbm, "us": tot_us,
            "traffic": {"encode_base_kernel": _kernel_traffic("encode_base_kernel"),
                        "encode_residual_kernel": _kernel_traffic("encode_residual_kernel")},
            "launches": out}


def run_deep(device, hbm, warmup=3, steps=10):
    """The 32-loop workload (one 16-head layer at N = 8192, R = 32 loops, geometric
    retention, 10 % key retention from loop 3): whole decode steps through the step
    executor with per-loop CUDA events, the algorithmic bytes of each loop taken from an
    untimed calibration step's selections; the loops <= 8 run the persistent sparse reader,
    loops 9..32 the direct one.  Plus the dense reader at loop 32 alone (the direct dense
    form: every column with its residual rows of loops 2..32)."""
    w = synth.WORKLOADS["deep_r32_h16_n8192"]
    R, H = w.loops, w.heads
    cache, wr = build_cache(w, 1, 0, device, new_tokens=warmup + steps + 1)
    inputs = step_inputs(wr, 1, warmup + steps + 1, device)
    O = torch.zeros(R + 1, 1, H, 128, dtype=torch.float32, device=device)
    # calibration step (untimed): loop by loop, the bytes each loop's launch moves
    q, kn, vn = inputs[0]
    cache.begin_token()
    k_sel = wr.k_sel(cache.n_cols)
    loop_bytes = {}
    for r in range(1, R + 1):
        cache.step(wr.dense_loops, k_sel, q, O, kn, vn, loop_first=r, loop_last=r, flush=cache.n_tail == 64)
        torch.cuda.synchronize()
        if r <= wr.dense_loops:
            res_rows = sum(cache.n_rows[0][rp] for rp in range(2, r + 1))
            loop_bytes[r] = bytemodel.dense_bytes(H, cache.n_q, cache.n_tail, res_rows, r == wr.dense_loops)
        else:
            loop_bytes[r] = sparse_bytes_from_state(cache, wr, 1, r, k_sel)
    ev_names = [f"e{i}" for i in range(2 * R + 1)]
    seg = {r: [] for r in range(1, R + 1)}
    sel = {r: [] for r in range(1, R + 1)}
    step_us = []
    for s in range(1, warmup + steps + 1):
        q, kn, vn = inputs[s]
        cache.begin_token()
        evs = [torch.cuda.Event(enable_timing=True) for _ in ev_names]
        cache.step(wr.dense_loops, wr.k_sel(cache.n_cols), q, O, kn, vn, events=evs, flush=cache.n_tail == 64)
        torch.cuda.synchronize()
        if s > warmup:
            step_us.append(evs[0].elapsed_time(evs[2 * R]) * 1e3)
            for r in range(1, R + 1):
                seg[r].append(evs[2 * r - 1].elapsed_time(evs[2 * r]) * 1e3)
                sel[r].append(evs[2 * r - 2].elapsed_time(evs[2 * r - 1]) * 1e3)
    st, info = cache.status()
    if st != 0:
        raise RuntimeError(f"device error in the deep-loop measurement: {info}")
    us = {r: float(np.mean(seg[r])) for r in range(1, R + 1)}
    groups = {"dense loops 1-2 (dense_staged_kernel)": range(1, wr.dense_loops + 1),
              "sparse loops 3-8 (sparse_persist_kernel)": range(wr.dense_loops + 1, 9),
              "sparse loops 9-32 (sparse_kernel, direct)": range(9, R + 1)}
    out = {}
    for name, rr in groups.items():
        b = sum(loop_bytes[r] for r in rr)
        t = sum(us[r] for r in rr)
        out[name] = {"us": t, "bytes": b, "achieved": b / (t * 1e-6) / 1e9, "frac": b / (t * 1e-6) / 1e9 / hbm,
                     "launches": len(rr)}
    sel_us = sum(float(np.mean(sel[r])) for r in range(wr.dense_loops + 1, R + 1))
    # the direct dense reader: full attention at loop 32 over every column (one launch)
    o = torch.empty(H, 128, dtype=torch.float32, device=device)
    qd = inputs[0][0][R][0].contiguous()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dts = []
    for rep in range(6):
        a.record()
        cache.dense(0, R, qd, o, keep_scores=False)
        b.record()
        torch.cuda.synchronize()
        if rep:
            dts.append(a.elapsed_time(b) * 1e3)
    d_us = float(np.mean(dts))
    d_bytes = bytemodel.dense_bytes(H, cache.n_q, cache.n_tail, sum(cache.n_rows[0][rp] for rp in range(2, R + 1)),
                                    False)
    total_b = sum(loop_bytes.values())
    step_mean = float(np.mean(step_us))
    del cache, inputs, O
    torch.cuda.empty_cache()
    return {"bound": "hbm", "workload": "deep_r32_h16_n8192 (1 layer, 16 heads, N=8192, R=32)",
            "us_per_step": step_mean, "bytes_per_step": total_b, "achieved": total_b / (step_mean * 1e-6) / 1e9,
            "peak": hbm, "unit": "GB/s", "frac": total_b / (step_mean * 1e-6) / 1e9 / hbm,
            "select_us_per_step": sel_us, "readers": out,
            "dense_direct_loop32": {"kernel": "dense_direct_kernel", "us_per_launch": d_us, "bytes_per_launch": d_bytes,
                                    "achieved": d_bytes / (d_us * 1e-6) / 1e9,
                                    "frac": d_bytes / (d_us * 1e-6) / 1e9 / hbm},
            "traffic": {"sparse_kernel": _kernel_traffic("sparse_kernel"),
                        "dense_direct_kernel": _kernel_traffic("dense_direct_kernel")}}


def _tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "of measured"
    except Exception:
        return 1590.0, "of fallback"


def run_prefill(w, device, reps=5):
    """Sparse prefill attention (fl_prefill_attn_sparse) on the workload's prompt: the loop-3
    active tokens (25 %) of every head attend causally over all tokens, BF16 K/V of
    H x N x 128.  Algorithmic FLOPs = 4 x 128 x (pos_i + 1) per active query and head (QK^T
    and PV, two per multiply-add, masked keys not counted); CUDA events on the launch stream
    after warm-up, inputs (2 x 134 MB of K/V) larger than L2."""
    from quantized_kv_attention_int4_b200 import abi

    n, H = w.n_ctx, w.heads
    pos = synth.active_sets(w, n)[3].to(torch.int32)
    g = torch.Generator(device=device).manual_seed(w.seed)
    k = torch.randn(H, n, 128, generator=g, device=device).to(torch.bfloat16)
    v = torch.randn(H, n, 128, generator=g, device=device).to(torch.bfloat16)
    q = torch.randn(H, pos.numel(), 128, generator=g, device=device).to(torch.bfloat16)
    o = torch.empty(H, pos.numel(), 128, dtype=torch.float32, device=device)
    pos_d = pos.to(device)
    flops = 4.0 * 128 * H * float((pos.to(torch.float64) + 1).sum())
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ts = []
    for rep in range(reps + 2):
        ev[0].record()
        abi.fl_prefill_attn_sparse(q, pos_d, k, v, o)
        ev[1].record()
        torch.cuda.synchronize()
        if rep >= 2:
            ts.append(ev[0].elapsed_time(ev[1]) * 1e3)
    us = float(np.mean(ts))
    tf = flops / (us * 1e-6) / 1e12
    peak, kind = _tensor_peak()
    del q, k, v, o
    return {"bound": "tensor", "kernel": f"prefill_attn_kernel (tcgen05; {pos.numel()} of {n} tokens active, {H} heads)",
            "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak, "peak_kind": kind,
            "traffic": None, "flops_per_launch": flops, "us_per_launch": us}


def run_e2e(step, cache, w, layers, inputs, device):
    """The metric end to end through the C ABI's host-buffer entry point (fl_decode_step_io):
    each step runs loops 1-3 untimed, then times one call that copies the loop-4 q / k_new /
    v_new from pinned host memory (one 2-D copy), runs the loop-4 selection and sparse
    readers, and copies the loop-4 outputs back to pinned host memory."""
    R, H = w.loops, w.heads
    qkv = torch.empty(3, R + 1, layers, H, 128, dtype=torch.bfloat16, device=device)
    hout = torch.empty(1, layers, H, 128, dtype=torch.float32).pin_memory()
    res, parts = [], []
    for q, kn, vn in inputs:
        hin = torch.stack([q[4], kn[4], vn[4]])[:, None].cpu().pin_memory()   # [3][1][L][H][128]
        qkv[0].copy_(q)
        qkv[1].copy_(kn)
        qkv[2].copy_(vn)
        qkv[:, 4].zero_()                        # loop 4's inputs arrive from the host
        step.run(qkv[0], qkv[1], qkv[2], loop_first=1, loop_last=3)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c = step.c
        a.record()
        c.step_io(w.dense_loops, w.k_sel(c.n_cols), qkv, hin, step.O, hout, loop_first=4, loop_last=4,
                  flush=c.n_tail == 64)
        b.record()
        b.synchronize()
        res.append(a.elapsed_time(b) * 1e3)
        assert torch.equal(hout[0], step.O[4].cpu())
    h2d = 3 * layers * H * 128 * 2
    d2h = layers * H * 128 * 4
    return {"value": float(np.mean(res)), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "api": "fl_decode_step_io (one call: host -> device copy, loop 4, device -> host copy); the timed "
                   "region starts before the call, so it includes the call's host-side time"}


# ----------------------------------------------------------------------------
# the oracle on the host cores
# ----------------------------------------------------------------------------
class OracleLoop4:
    """The oracle's loop-4 selection + sparse attention for one (layer, head) sample.

    Construction (untimed) encodes the prompt and runs loops 1-3; `run_once()` times one
    loop-4 step (top-K selection from the spliced distribution, then the sparse loop)
    from the same state and returns its seconds per (layer, head).
    """

    def __init__(self, w: synth.Workload, heads=(0,), codec: int = 0):
        from oracle import flashloop_oracle as fo

        self.fo = fo
        n = w.n_ctx
        sets = synth.active_sets(w, n)
        d = synth.prefill_layer(w, 0, device="cpu", sets=sets)
        n_q, n_tail = synth.split_prefill(n)
        hs = list(heads)
        self.nh = len(hs)
        f = lambda t: t.float().numpy()
        lay = fo.OracleLayer(len(hs), w.loops, n + 64, codec=codec)
        lay.encode_base(0, f(d["K"][1][hs, :n_q]), f(d["V"][1][hs, :n_q]))
        for r in range(2, w.loops + 1):
            rows = sets[r][sets[r] < n_q].numpy()
            lay.encode_residual(r, rows, f(d["K"][r][hs][:, rows]), f(d["V"][r][hs][:, rows]))
        depth = synth.depth_of(sets, n).numpy()
        lay.set_tail([None] + [f(d["K"][r][hs, n_q:]) for r in range(1, w.loops + 1)],
                     [None] + [f(d["V"][r][hs, n_q:]) for r in range(1, w.loops + 1)], depth[n_q:])
        del d
        self.q = synth.queries(w, 0, 0).float().numpy()[:, hs]
        self.k = w.k_sel(lay.n_cols)
        for r in range(1, 4):
            if r <= w.dense_loops:
                lay.dense_loop(r, self.q[r])
            else:
                S, _, _ = lay.select(self.k)
                lay.sparse_loop(r, self.q[r], S)
        self.lay = lay
        self.p_save, self.lam_save = lay.p_tilde.copy(), lay.lam.copy()

    def run_once(self) -> float:
        """One timed loop-4 step on a single host thread (BLAS pool limited to 1)."""
        from threadpoolctl import threadpool_limits

        lay = self.lay
        lay.p_tilde, lay.lam = self.p_save.copy(), self.lam_save.copy()
        with threadpool_limits(limits=1):
            t = time.perf_counter()
            S = self.fo.select_topk(lay.p_tilde, self.k)
            lay.sparse_loop(4, self.q[4], S)
            dt = time.perf_counter() - t
        return dt / self.nh


def oracle_loop4_sample(w: synth.Workload, budget_s: float, heads=(0,)):
    """Seconds per (layer, head) of the oracle's loop-4 step, averaged over repetitions
    that fill about ``budget_s`` seconds; returns (seconds, repetitions)."""
    o = OracleLoop4(w, heads)
    times = []
    t_all = time.perf_counter()
    while True:
        times.append(o.run_once())
        if time.perf_counter() - t_all > budget_s and len(times) >= 2:
            break
    return float(np.mean(times)), len(times)


def oracle_beside(w: synth.Workload, layers: int, codec_layers: int, budget_s: float, rows=None):
    """The oracle timed beside the rows measured outside the decode steps, on one host thread,
    each on a bounded sample of the GPU leg's workload (seeded CPU inputs of the same shapes
    and distributions): the token-sparse update selector (loop-3 ranking, every token), the
    sparse prefill attention (the 64 latest active queries of one head, scaled by FLOPs) and
    the loop-4 step of each codec variant (one (layer, head), scaled like cpu_baseline)."""
    from threadpoolctl import threadpool_limits
    from oracle import flashloop_oracle as fo

    out = {}
    n, d = w.n_ctx, w.heads * 128
    ns = n // 8                          # a bounded sample: an eighth of the tokens, scaled by 8
    rng = np.random.default_rng(w.seed)
    h1 = rng.standard_normal((ns, d), dtype=np.float32)
    h2 = (h1 + rng.standard_normal((ns, d), dtype=np.float32) * np.exp(rng.standard_normal((ns, 1)))).astype(np.float32)
    k3 = w.n_active(3, ns)
    with threadpool_limits(limits=1):
        fo.select_active(h1, h2, np.arange(ns), k3)          # untimed: first-touch of the buffers
        t = time.perf_counter()
        fo.select_active(h1, h2, np.arange(ns), k3)
        dt = time.perf_counter() - t
    out["token_select"] = {"value": dt * (n / ns) * 1e6, "unit": "us per loop-3 ranking", "cores": 1,
                           "kind": "oracle",
                           "sample": f"oracle select_active over {ns} of {n} tokens x {d} (fp64), scaled by {n // ns}"}
    del h1, h2
    pos = synth.active_sets(w, n)[3].numpy()
    sample = pos[-64:]
    K = rng.standard_normal((1, n, 128), dtype=np.float32)
    V = rng.standard_normal((1, n, 128), dtype=np.float32)
    q = rng.standard_normal((1, sample.size, 128), dtype=np.float32)
    with threadpool_limits(limits=1):
        fo.prefill_attention(q[:, :4], sample[:4], K, V)      # untimed: first-touch of the buffers
        t = time.perf_counter()
        fo.prefill_attention(q, sample, K, V)
        dt = time.perf_counter() - t
    scale = w.heads * float((pos.astype(np.float64) + 1).sum()) / float((sample.astype(np.float64) + 1).sum())
    out["prefill"] = {"value": dt * scale * 1e6, "unit": "us per call", "cores": 1, "kind": "oracle",
                      "sample": f"oracle prefill_attention for the 64 latest of {pos.size} active queries of 1 of "
                                f"{w.heads} heads (fp64), scaled by FLOPs x{scale:.0f}"}
    del K, V, q
    for codec, name in ((fo.FULL_INT4, "full_int4"), (fo.RESIDUAL_INT2, "residual_int2")):
        o = OracleLoop4(w, codec=codec)
        times = []
        t_all = time.perf_counter()
        while not times or (time.perf_counter() - t_all < budget_s and len(times) < 50):
            times.append(o.run_once())
        out[name] = {"value": float(np.mean(times)) * codec_layers * w.heads * 1e6, "unit": "us per loop-4 step",
                     "cores": 1, "kind": "oracle",
                     "sample": f"oracle loop-4 selection + sparse attention, {name} stores, 1 of {codec_layers}x"
                               f"{w.heads} (layer, head) pairs at N={n}, {len(times)} reps, scaled by "
                               f"{codec_layers * w.heads}"}
        del o
    return out


def _oracle_worker(args):
    """One host core's share of the all-cores baseline (a spawned process, one BLAS thread):
    set up the oracle's state for one (layer, head) of the workload, then time loop-4 steps
    for about `budget_s` seconds.  Returns (seconds per step, repetitions)."""
    name, head, budget_s = args
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=1):
        o = OracleLoop4(synth.WORKLOADS[name], heads=(head,))
        times = []
        t_all = time.perf_counter()
        while not times or (time.perf_counter() - t_all < budget_s and len(times) < 200):
            times.append(o.run_once())
    return float(np.mean(times)), len(times)


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w: synth.Workload, layers: int, budget_s: float):
    """The oracle's loop-4 step (top-K selection + sparse attention) on the host cores: the
    single-thread figure, and every core at once (one spawned process per core, each with
    its own (layer, head) sample and one BLAS thread), scaled to the workload's layers x
    heads pairs by the pairs a second the cores finish together."""
    import multiprocessing as mp

    per_lh, reps = oracle_loop4_sample(w, budget_s)
    single_us = per_lh * layers * w.heads * 1e6
    cores = host_cores()
    pairs = layers * w.heads
    with mp.get_context("spawn").Pool(cores) as pool:
        res = pool.map(_oracle_worker, [(w.name, i % w.heads, budget_s) for i in range(cores)])
    per_pair = float(np.mean([t for t, _ in res]))      # seconds per pair on one core, all cores busy
    all_us = pairs * per_pair / cores * 1e6
    return {"value": all_us, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"oracle (NumPy, fp64) loop-4 top-K selection + sparse attention at N={w.n_ctx}: "
                      f"{cores} processes at once, one (layer, head) pair each ({sum(n for _, n in res)} steps), "
                      f"scaled to {layers}x{w.heads} pairs shared by {cores} cores",
            "single_thread": {"value": single_us, "unit": UNIT, "cores": 1,
                              "sample": f"1 of {pairs} (layer, head) pairs, {reps} reps, scaled by {pairs}"}}


_REF_STATE = {}


def _ref_init(name, head):
    from threadpoolctl import threadpool_limits

    threadpool_limits(limits=1)
    _REF_STATE["o"] = OracleLoop4(synth.WORKLOADS[name], heads=(head,))


def _ref_step(_):
    return _REF_STATE["o"].run_once()


def reference_arm(w: synth.Workload, layers: int, args, config) -> dict:
    """The oracle as the reference arm, on every host core: one spawned process per core,
    each holding one (layer, head) pair's state; a step is one loop-4 step (top-K selection
    + sparse attention) on every process at once, scaled to the workload's layers x heads
    pairs shared by the cores."""
    import multiprocessing as mp

    cores = host_cores()
    pairs = layers * w.heads
    ctx = mp.get_context("spawn")
    per_step = []
    # each process sets up its own pair: the initializer draws a distinct head per process
    with ctx.Pool(cores, initializer=_ref_init_next, initargs=(w.name, w.heads, ctx.Value("i", 0))) as pool:
        for _ in range(args.warmup + args.steps):
            t = pool.map(_ref_step, range(cores), chunksize=1)
            per_step.append(pairs * float(np.mean(t)) / cores * 1e6)
    v = float(np.mean(per_step[args.warmup:]))
    return {"metric": METRIC, "value": v, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"oracle loop-4 selection + sparse attention, {cores} processes at once with "
                                       f"one (layer, head) pair each per step, scaled to {pairs} pairs shared by "
                                       f"{cores} cores"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def _ref_init_next(name, n_heads, counter):
    with counter.get_lock():
        i = counter.value
        counter.value += 1
    _ref_init(name, i % n_heads)


# ----------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("flashloop", "reference"), default="flashloop")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--layers", type=int, default=0, help="override the workload's layer count")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-token-select", dest="token_select", action="store_false",
                    help="skip the token-sparse update selector measurement")
    ap.add_argument("--no-prefill", dest="prefill", action="store_false",
                    help="skip the sparse prefill attention measurement")
    ap.add_argument("--no-codecs", dest="codecs", action="store_false",
                    help="skip the codec variant (full-state INT4, INT2 residual) measurement")
    ap.add_argument("--codec-layers", type=int, default=4, help="layers of each codec variant's cache")
    ap.add_argument("--no-encode", dest="encode", action="store_false",
                    help="skip the prefill encode measurement (one 32K layer)")
    ap.add_argument("--no-deep", dest="deep", action="store_false",
                    help="skip the 32-loop workload measurement")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = synth.WORKLOADS[args.workload]
    layers = args.layers or w.layers
    config = {"workload": args.workload, "layers": layers, "heads": w.heads, "head_dim": 128,
              "context": w.n_ctx, "loops": w.loops, "dense_loops": w.dense_loops, "key_pct": w.key_pct,
              "retention": "100/100/25/10 %", "storage": "int4 base+residual, bf16 tail",
              "l2": "inputs larger than L2: loop-major over all layers, ~1.3 GB read between reuses of a layer"}

    if args.impl == "reference":
        if rank != 0:
            return
        line = reference_arm(w, layers, args, config)
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)

    r = run_gpu(args, rank, world)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline(w, layers, args.cpu_budget)
        beside = oracle_beside(w, layers, args.codec_layers, 3.0)
        if r["tokens"]:
            r["tokens"]["cpu_baseline"] = beside["token_select"]
        if r["prefill"]:
            r["prefill"]["cpu_baseline"] = beside["prefill"]
        if r["codecs"]:
            for name, v in r["codecs"].items():
                v["cpu_baseline"] = beside[name]
    hbm = r["hbm"]
    sp_layer = _kernel_traffic("sparse_persist_kernel")   # ncu DRAM bytes per layer (8-layer capture)
    sp_traffic = sp_layer * r["layers"] if sp_layer is not None else None
    line = {
        "metric": METRIC, "value": r["metric_us"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["step_ms"], "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": {**config, "context_at_end": r["N"],
                                                                          "k_sel": r["k_sel"]},
        "roofline": {"bound": "hbm", "kernel": "sparse_persist_kernel (loop 4: one launch for every layer, then "
                               "its combine)", "achieved": r["sp_gbs"],
                     "peak": hbm, "unit": "GB/s", "frac": r["sp_gbs"] / hbm, "traffic": sp_traffic,
                     "peak_kind": peak_kind_str(r["peak_kind"]), "bytes_per_launch": r["sp_bytes"] * r["layers"],
                     "us_per_launch": r["sp_launch_us"] * r["layers"], "layers_per_launch": r["layers"],
                     "bytes_per_layer": r["sp_bytes"], "us_per_layer": r["sp_launch_us"]},
        "roofline_dense": {"bound": "hbm", "kernel": "fl_decode_attn_dense (loops 1-2)", "achieved": r["d_gbs"],
                           "peak": hbm, "unit": "GB/s", "frac": r["d_gbs"] / hbm, "traffic": _kernel_traffic("dense_staged_kernel"),
                           "bytes_per_launch": r["d_bytes"], "us_per_launch": r["d_launch_us"]},
        "roofline_encode": r["encode"],
        "roofline_cfg4": r["deep"],
        "roofline_token_select": r["tokens"],
        "roofline_prefill": r["prefill"],
        "codec_variants": r["codecs"],
        "segments_ms": r["seg"], "clocks": r["clocks"], "gpu_launches": r["launches"],
        "e2e": r["e2e"], "cpu_baseline": cpu, "setup_s": r["setup_s"],
    }
    print(json.dumps(line), flush=True)


def peak_kind_str(kind):
    return "of measured" if kind == "measured" else "of fallback"


if __name__ == "__main__":
    main()

"""Test-side helpers: unpack the library's packed cache into logical arrays, build a
GPU cache and an oracle from the same synthetic inputs, and compare them."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import flashloop_oracle as fo
from quantized_kv_attention_int4_b200 import abi
from quantized_kv_attention_int4_b200.cache import FlashLoopCache, round_up, split_prefill

TOL = 2e-3


def f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def nibbles(raw: np.ndarray) -> np.ndarray:
    """[..., 64] packed bytes -> [..., 128] codes (byte b = channels 2b low, 2b+1 high)."""
    out = np.empty(raw.shape[:-1] + (raw.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = raw & 15
    out[..., 1::2] = raw >> 4
    return out


def split_sz(raw: np.ndarray):
    """uint32 (scale | zero << 16) -> (scale f16, zero f16)."""
    return (raw & 0xFFFF).astype(np.uint16).view(np.float16), (raw >> 16).astype(np.uint16).view(np.float16)


def _split_records(raw: np.ndarray, H: int, G: int):
    """Group records [H][G][9216] -> key codes, value codes [H][G*64][128], key sz [H][G][128], value sz [H][G*64][2]."""
    rec = raw[: H * G * 9216].reshape(H, G, 9216)
    rows = rec[:, :, :8192].reshape(H, G, 64, 128)
    kc = nibbles(rows[..., :64].reshape(H, G * 64, 64))
    vc = nibbles(rows[..., 64:].reshape(H, G * 64, 64))
    vsz = np.ascontiguousarray(rec[:, :, 8192:8704]).view(np.uint32).reshape(H, G * 64, 2)
    ksz = np.ascontiguousarray(rec[:, :, 8704:]).view(np.uint32).reshape(H, G, 128)
    return kc, vc, ksz, vsz


def crumbs(words: np.ndarray) -> np.ndarray:
    """[..., 8] uint32 words of 2-bit codes -> [..., 128] codes.

    Word w holds channels 16w .. 16w+15: channel 16w+k (k < 8) in bits 4k..4k+1 and
    channel 16w+8+k in bits 4k+2..4k+3 (include/flashloop.h, 2-bit residual records)."""
    out = np.empty(words.shape[:-1] + (words.shape[-1], 16), np.uint8)
    for k in range(8):
        out[..., k] = (words >> (4 * k)) & 3
        out[..., 8 + k] = (words >> (4 * k + 2)) & 3
    return out.reshape(words.shape[:-1] + (words.shape[-1] * 16,))


def _split_records2(raw: np.ndarray, H: int, G: int):
    """2-bit residual records [H][G][5120] -> the same logical arrays as _split_records."""
    rec = raw[: H * G * 5120].reshape(H, G, 5120)
    rows = np.ascontiguousarray(rec[:, :, :4096]).reshape(H, G * 64, 64)
    kc = crumbs(np.ascontiguousarray(rows[..., :32]).view(np.uint32))
    vc = crumbs(np.ascontiguousarray(rows[..., 32:]).view(np.uint32))
    vsz = np.ascontiguousarray(rec[:, :, 4096:4608]).view(np.uint32).reshape(H, G * 64, 2)
    ksz = np.ascontiguousarray(rec[:, :, 4608:]).view(np.uint32).reshape(H, G, 128)
    return kc, vc, ksz, vsz


class Unpacked:
    """Logical views of one layer of a FlashLoopCache (CPU copies)."""

    def __init__(self, cache: FlashLoopCache, layer: int = 0):
        H, C, R = cache.H, cache.capacity, cache.R
        T = cache.layout.total_slots
        g = lambda n: cache.raw(n, layer).cpu().numpy()
        self.kc, self.vc, ksz, vsz = _split_records(g("brec"), H, C // 64)
        self.ks, self.kz = split_sz(ksz)
        self.vs, self.vz = split_sz(vsz)
        split = _split_records2 if cache.codec == abi.FL_CODEC_RESIDUAL_INT2 else _split_records
        self.rkc, self.rvc, rksz, rvsz = split(g("rrec"), H, T // 64)
        self.rks, self.rkz = split_sz(rksz)
        self.rvs, self.rvz = split_sz(rvsz)
        self.mask = g("mask").view(np.uint64)[: (R + 1) * (C // 64)].reshape(R + 1, C // 64)
        self.first = g("first").view(np.int32)[: (R + 1) * (C // 64)].reshape(R + 1, C // 64)
        self.depth = g("depth")[:C]
        self.slot_base = list(cache.layout.slot_base)


def selection(cache: FlashLoopCache, layer: int, k_sel: int):
    H, ms = cache.H, cache.dims.max_select
    S = cache.raw("sel", layer).view(torch.int32)[: H * ms].view(H, ms)[:, :k_sel].cpu().numpy().astype(np.int64)
    m = cache.raw("mass", layer).view(torch.float32)[:H].cpu().numpy().astype(np.float64)
    u = cache.raw("unsel", layer).view(torch.float32)[: H * 128].view(H, 128).cpu().numpy().astype(np.float64)
    return S, m, u


def rel_err(got, ref) -> float:
    """Max over heads (first axis) of ||got - ref||_inf / ||ref||_inf."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.abs(got - ref).reshape(ref.shape[0], -1).max(axis=1)
    den = np.abs(ref).reshape(ref.shape[0], -1).max(axis=1)
    return float((num / np.maximum(den, 1e-30)).max())


# Elementwise relative errors seen by the parity tests, reported at the end of the run
# (conftest.py): |got - ref| / max(|ref|, 1e-3 ||ref||_inf) per head, the floor keeping
# near-zero reference entries from dominating.
ELEMENTWISE: dict = {}
ELEM_FLOOR = 1e-3
ELEM_BOUND = 1e-2


def u_err(u, u_ref, o_prev, o_prev_ref) -> float:
    """Error of the unselected contribution u against ||u_ref||_inf per head, beyond the
    error it inherits from the previous loop's output.

    The readers form u = o_prev - sum_S p~_j v_j from the previous loop's output, so
    whatever error o_prev carries (each loop's own output is held to 2e-3 of its norm,
    in practice ~1e-6) passes into u unchanged; when the selected mass m approaches 1,
    ||u|| is far below ||o_prev|| and that inherited part dominates a relative measure.
    This returns max over heads of max(0, ||u - u_ref|| - ||o_prev - o_prev_ref||) /
    ||u_ref||; ELEMENTWISE keeps the plain relative error for the report."""
    u, u_ref = np.asarray(u, np.float64), np.asarray(u_ref, np.float64)
    inh = np.abs(np.asarray(o_prev, np.float64) - np.asarray(o_prev_ref, np.float64)).max(axis=1)
    num = np.maximum(np.abs(u - u_ref).max(axis=1) - inh, 0.0)
    den = np.maximum(np.abs(u_ref).max(axis=1), 1e-30)
    return float((num / den).max())


def elem_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    H = ref.shape[0]
    g, r = got.reshape(H, -1), ref.reshape(H, -1)
    floor = ELEM_FLOOR * np.abs(r).max(axis=1, keepdims=True)
    return float((np.abs(g - r) / np.maximum(np.abs(r), np.maximum(floor, 1e-30))).max())


def note_elementwise(label: str, got, ref) -> float:
    if not np.abs(np.asarray(ref)).max() > 0:   # an exactly zero reference has no relative error
        return 0.0
    e = elem_err(got, ref)
    ELEMENTWISE[label] = max(ELEMENTWISE.get(label, 0.0), e)
    return e


def check_topk_valid(S, p_tilde, k):
    """S (per head, ascending, unique) is a top-k of p_tilde up to tau = 1e-5 * max p_tilde."""
    H, N = p_tilde.shape
    for h in range(H):
        s = S[h]
        assert s.shape == (k,) and np.all(np.diff(s) > 0) and s[0] >= 0 and s[-1] < N
        tau = 1e-5 * p_tilde[h].max()
        inside = np.zeros(N, bool)
        inside[s] = True
        if k < N:
            assert p_tilde[h][inside].min() >= p_tilde[h][~inside].max() - tau


class Pair:
    """A one-layer GPU cache and its oracle, built from the same synthetic prompt."""

    def __init__(self, w: synth.Workload, heads=None, extra_tokens: int = 0, layer: int = 0, data=None,
                 codec: int = abi.FL_CODEC_RESIDUAL_INT4):
        self.w = w
        self.layer = layer
        n = w.n_ctx
        self.heads = list(range(w.heads)) if heads is None else list(heads)
        cap = round_up(n + extra_tokens + 64)
        self.cache = FlashLoopCache(1, w.heads, w.loops, cap, max_select=cap, codec=codec)
        d = synth.prefill_layer(w, layer, device="cuda") if data is None else data
        self.sets = d["sets"]
        n_q, n_tail, tail_depth = self.cache.prefill_layer(0, d["K"], d["V"], self.sets)
        self.cache.set_timeline(n_q, n_tail, tail_depth)
        hs = self.heads
        self.oracle = fo.OracleLayer(len(hs), w.loops, cap, codec=codec)
        lay = self.oracle
        lay.encode_base(0, f32(d["K"][1][hs, :n_q]), f32(d["V"][1][hs, :n_q]))
        self.calls = {r: [] for r in range(2, w.loops + 1)}
        for r in range(2, w.loops + 1):
            rows = self.sets[r][self.sets[r] < n_q].numpy()
            lay.encode_residual(r, rows, f32(d["K"][r][hs][:, rows]), f32(d["V"][r][hs][:, rows]))
            self.calls[r].append((0, len(rows)))
        lay.set_tail([None] + [f32(d["K"][r][hs, n_q:]) for r in range(1, w.loops + 1)],
                     [None] + [f32(d["V"][r][hs, n_q:]) for r in range(1, w.loops + 1)], np.array(tail_depth))
        del d

    # -- decode --------------------------------------------------------------------
    def _note_flush(self):
        """The residual slots a flush of the current full tail takes (for compare_encoding)."""
        for r in range(2, self.w.loops + 1):
            slot0 = round_up(self.cache.n_slots[0][r])
            self.calls[r].append((slot0, sum(1 for dep in self.cache.tail_depth if dep >= r)))

    def begin_token(self, step: int):
        """Append decode token ``step`` (flushing a full tail first) on both sides."""
        w, hs = self.w, self.heads
        if self.cache.n_tail == 64:
            self._note_flush()
        self.cache.begin_token()
        tok = synth.decode_token(w, self.layer, step, device="cuda")
        self.oracle.append_token([None] + [f32(tok["k"][r][hs]) for r in range(1, w.loops + 1)],
                                 [None] + [f32(tok["v"][r][hs]) for r in range(1, w.loops + 1)])
        return tok

    def run_loops(self, q, tok=None, k_sel=None, loops=None, check=True, fused=False, oracle=True, label=None):
        """Every loop of one decode step on the GPU and in the oracle; returns per-loop errors.

        With ``fused`` the GPU side runs each loop through the step executor, and a full
        tail is flushed by the step's own readers (fl_decode_step_flush).  With
        ``oracle=False`` only the GPU side runs (the oracle's next dense loop starts its
        distribution afresh, so a skipped step leaves nothing stale).  Errors: o per loop,
        m, and u against ||u_ref||_inf; elementwise errors are noted under ``label``."""
        w, hs, c, lay = self.w, self.heads, self.cache, self.oracle
        H = w.heads
        N = c.n_cols
        k_sel = w.k_sel(N) if k_sel is None else k_sel
        errs = {}
        o_prev = None
        prev_ref = None
        flush = fused and c.n_tail == 64
        if fused:
            if flush:
                self._note_flush()
            R = w.loops
            Q = q[:, None].contiguous()
            O = torch.zeros(R + 1, 1, H, 128, dtype=torch.float32, device="cuda")
            zero = torch.zeros(H, 128, dtype=torch.bfloat16, device="cuda")
            KN = torch.stack([zero] + [tok["k"][r] for r in range(1, R + 1)])[:, None].contiguous() if tok else None
            VN = torch.stack([zero] + [tok["v"][r] for r in range(1, R + 1)])[:, None].contiguous() if tok else None
        for r in range(1, (loops or w.loops) + 1):
            o = torch.empty(H, 128, dtype=torch.float32, device="cuda")
            kn = tok["k"][r] if tok else None
            vn = tok["v"][r] if tok else None
            qr = q[r].contiguous()
            if fused:
                c.step(w.dense_loops, k_sel, Q, O, KN, VN, loop_first=r, loop_last=r, flush=flush)
                o = O[r, 0]
            if r <= w.dense_loops:
                if not fused:
                    c.dense(0, r, qr, o, kn, vn, keep_scores=True)
                if oracle:
                    ref = lay.dense_loop(r, f32(q[r][hs]))
                    got = o.cpu().numpy()[hs]
                    errs[r] = rel_err(got, ref["o"])
                    prev_ref = ref["o"]
                    if label:
                        note_elementwise(f"{label} o", got, ref["o"])
            else:
                if not fused:
                    c.select(0, 1, r, k_sel)
                if oracle:
                    S, _, _ = selection(c, 0, k_sel)
                    if check:
                        check_topk_valid(S[hs], lay.p_tilde, k_sel)
                if not fused:
                    c.sparse(0, r, k_sel, qr, o_prev, o, kn, vn)
                if oracle:
                    _, m, u = selection(c, 0, k_sel)
                    ref = lay.sparse_loop(r, f32(q[r][hs]), S[hs])
                    errs[(r, "m")] = float(np.max(np.abs(m[hs] - ref["m"]) / ref["m"]))
                    errs[(r, "u")] = u_err(u[hs], ref["u"], o_prev.cpu().numpy()[hs], prev_ref)
                    got = o.cpu().numpy()[hs]
                    errs[r] = rel_err(got, ref["o"])
                    prev_ref = ref["o"]
                    if label:
                        note_elementwise(f"{label} o", got, ref["o"])
                        note_elementwise(f"{label} u", u[hs], ref["u"])
                        if np.abs(ref["u"]).max(axis=1).min() > 0:
                            ELEMENTWISE[f"{label} u vs ||u||"] = max(ELEMENTWISE.get(f"{label} u vs ||u||", 0.0),
                                                                   rel_err(u[hs], ref["u"]))
            o_prev = o
        st, info = c.status()
        assert st == abi.FL_OK, info
        return errs


def compare_encoding(pair: Pair):
    """Codes, scales and zero points of base and residual stores are bit-exact; the
    block masks / first slots / depths address exactly the oracle's slots."""
    U = Unpacked(pair.cache)
    lay, hs, n_q = pair.oracle, pair.heads, pair.cache.n_q
    nb = n_q // 64
    u16 = lambda a: np.ascontiguousarray(a).view(np.uint16)
    assert np.array_equal(U.kc[hs, :n_q], lay.base["kc"][:, :n_q])
    assert np.array_equal(U.vc[hs, :n_q], lay.base["vc"][:, :n_q])
    assert np.array_equal(u16(U.ks[hs, :nb]), u16(lay.base["ks"][:, :nb]))
    assert np.array_equal(u16(U.kz[hs, :nb]), u16(lay.base["kz"][:, :nb]))
    assert np.array_equal(u16(U.vs[hs, :n_q]), u16(lay.base["vs"][:, :n_q]))
    assert np.array_equal(u16(U.vz[hs, :n_q]), u16(lay.base["vz"][:, :n_q]))
    assert np.array_equal(U.depth[:n_q], lay.depth[:n_q])
    for r in range(2, pair.w.loops + 1):
        assert len(pair.calls[r]) == len(lay.calls[r])
        for (slot0, n), call in zip(pair.calls[r], lay.calls[r]):
            enc = call["enc"]
            g0 = U.slot_base[r] + slot0
            ng = -(-n // 64)
            assert np.array_equal(U.rkc[hs, g0:g0 + n], enc["kc"])
            assert np.array_equal(U.rvc[hs, g0:g0 + n], enc["vc"])
            assert not U.rkc[hs, g0 + n:g0 + ng * 64].any()
            assert np.array_equal(u16(U.rks[hs, g0 // 64:g0 // 64 + ng]), u16(enc["ks"]))
            assert np.array_equal(u16(U.rkz[hs, g0 // 64:g0 // 64 + ng]), u16(enc["kz"]))
            assert np.array_equal(u16(U.rvs[hs, g0:g0 + n]), u16(enc["vs"]))
            assert np.array_equal(u16(U.rvz[hs, g0:g0 + n]), u16(enc["vz"]))
            rows = call["rows"]
            for i, j in enumerate(rows.tolist()):
                b, t = j // 64, j % 64
                mk = int(U.mask[r, b])
                assert (mk >> t) & 1
                assert U.first[r, b] + bin(mk & ((1 << t) - 1)).count("1") == slot0 + i
        act = lay.depth[:n_q] >= r
        bits = np.zeros(nb, np.uint64)
        for j in np.nonzero(act)[0].tolist():
            bits[j // 64] |= np.uint64(1 << (j % 64))
        assert np.array_equal(U.mask[r, :nb], bits)

"""FlashLoop decode-path oracle.  TEST INFRASTRUCTURE ONLY.

A plain, slow NumPy restatement of what the FlashLoop pages say the decode path
computes.  It is the yardstick the CUDA library is checked against and is never
part of the product path: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.  It
shares no code with the CUDA library and imports nothing from it.

Sources (page title, then section):

* [PyPI]    "flashloop 0.1.0" project description, "Configuration and supported
            scope": four loops, dense loops 1-2, 25 % / 10 % token retention in
            loops 3-4, 10 % key retention, 4-bit K/V, group 64, 64-token BF16 tail.
* [Project] "FlashLoop: Fast and Memory-Efficient Looped Transformers via Lazy
            Updates" project page, "The Method", Steps 01-03.
* [Guide]   flozi.net "FlashLoop: store changes between repeated passes",
            section 3 "What FlashLoop actually computes".
* [KIVI]    the KIVI lineage the guide cites for its conventions (keys grouped
            per channel along tokens, values per token along channels).

Readings where the pages are silent (each listed again in the design notes):

* quantiser: scale s = fp16(RN((max - min) / 15)) in fp32, zero z = fp16(min),
  code = clamp(rint((x - z) / s), 0, 15) with fp32 subtract/divide and
  round-half-even, code 0 for a zero-width group; dequantisation is the single
  rounding fma(code, s, z);
* residual key groups are 64 consecutive compact rows ("slots") of one encode
  call, per channel; a call's last group may be partial;
* codec variants (the ablations named in [Guide] section 4, the "Per-loop KIVI4"
  row and the 2-bit row of Figure 5, and the [Project] "Experiments" caption of
  Figure 5, right: residual precision varied): "per-loop KIVI4" stores each loop
  r >= 2 as INT4 codes of the full state X^(r) of its active rows (grouped like the
  residual stores), and a token's loop-r state is then that one store, the one of
  loop min(r, depth); "INT2 residuals" keeps the INT4 base and quantises the
  residuals with 2-bit codes, s = fp16((max - min) / 3);
* the BF16 tail holds the most recent 1..64 columns of every loop;
* token-sparse updates rank the tokens of A_{r-1} by the squared relative L2 change
  ||h^(r-1) - h^(r-2)||^2 / ||h^(r-2)||^2 of their hidden state over loop r-1, in
  fp64, ties to the lower token;
* sparse loop r re-selects from the spliced distribution of loop r-1, ties go
  to the smaller column index, and its output is
  o_r = u + m * softmax_S(q K_S^T / sqrt(d)) V_S with m the selected mass and u
  the unselected columns' contribution, each column at the loop that last
  computed it.

Every function is pinned by a ``-m "not gpu"`` test (closed forms, brute force,
invariants); none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

F16 = np.float16
F32 = np.float32
F64 = np.float64
HEAD_DIM = 128
GROUP = 64
TAIL = 64
LEVELS = 15  # 4-bit codes 0..15
LEVELS2 = 3  # 2-bit codes 0..3

# Codecs of the loop r >= 2 stores (the base is always 4-bit):
RESIDUAL_INT4 = 0  # X^(r) - X_hat^(r-1), 4-bit (the method)
FULL_INT4 = 1      # X^(r) itself, 4-bit ("per-loop KIVI4")
RESIDUAL_INT2 = 2  # X^(r) - X_hat^(r-1), 2-bit


# ----------------------------------------------------------------------------
# 4-bit asymmetric group codec  ([PyPI] "4-bit K/V, group size 64";
# [Guide] section 3 "group-wise asymmetric, group 64")
# ----------------------------------------------------------------------------
def half_rn(x) -> np.ndarray:
    """fp32 -> IEEE binary16, round to nearest, ties to even."""
    return np.asarray(x, dtype=F32).astype(F16)


def quantize(x, axis: int = -1, levels: int = LEVELS):
    """Quantise every group laid out along ``axis`` to codes 0 .. levels (15: 4-bit).

    Returns (codes uint8 with x's shape, scale fp16, zero fp16) where scale and
    zero have ``axis`` removed.  Arithmetic is fp32 with one rounding per
    operation: s = fp16((max - min) / levels), z = fp16(min),
    code = clamp(rint((x - z) / s), 0, levels), and 0 when s is zero.
    """
    x = np.moveaxis(np.asarray(x, dtype=F32), axis, -1)
    mn = x.min(axis=-1)
    mx = x.max(axis=-1)
    s = half_rn(np.subtract(mx, mn, dtype=F32) / F32(levels))
    z = half_rn(mn)
    sf = s.astype(F32)[..., None]
    zf = z.astype(F32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.subtract(x, zf, dtype=F32) / sf
    codes = np.clip(np.rint(t), 0, levels)
    codes = np.where(sf == 0, F32(0), codes)
    return np.moveaxis(codes.astype(np.uint8), -1, axis), s, z


def dequant(codes, s, z) -> np.ndarray:
    """x_hat = fma(code, s, z) rounded once to fp32.

    code * s and the sum are exact in fp64 for binary16 s and z, so the single
    final rounding equals a correctly rounded fp32 fused multiply-add.
    """
    return (np.asarray(codes, F64) * np.asarray(s, F64) + np.asarray(z, F64)).astype(F32)


# ----------------------------------------------------------------------------
# Base (loop 1) and residual (loop r >= 2) encoders  ([Project] Step 03;
# [Guide] section 3: per-channel keys, per-token values, residual
# X^(r) - X_hat^(r-1) of active tokens only)
# ----------------------------------------------------------------------------
def encode_base(K, V) -> dict:
    """Quantise loop-1 keys and values of T tokens (T a multiple of 64).

    K, V: fp32 [H][T][128].  Keys: one group per (64-token block, channel).
    Values: one group per (token, 64-channel half).
    Returns kc/vc uint8 [H][T][128], ks/kz fp16 [H][T/64][128], vs/vz fp16 [H][T][2].
    """
    K = np.asarray(K, F32)
    V = np.asarray(V, F32)
    H, T, D = K.shape
    assert D == HEAD_DIM and T % GROUP == 0
    kc, ks, kz = quantize(K.reshape(H, T // GROUP, GROUP, D), axis=2)
    vc, vs, vz = quantize(V.reshape(H, T, 2, D // 2), axis=3)
    return dict(kc=kc.reshape(H, T, D), ks=ks, kz=kz, vc=vc.reshape(H, T, D), vs=vs, vz=vz)


def decode_base(enc: dict):
    """Dequantised (K_hat, V_hat) fp32 [H][T][128] of an encode_base result."""
    H, T, D = enc["kc"].shape
    kh = dequant(enc["kc"].reshape(H, T // GROUP, GROUP, D), enc["ks"][:, :, None, :],
                 enc["kz"][:, :, None, :]).reshape(H, T, D)
    vh = dequant(enc["vc"].reshape(H, T, 2, D // 2), enc["vs"][..., None],
                 enc["vz"][..., None]).reshape(H, T, D)
    return kh, vh


def encode_residual(EK, EV, levels: int = LEVELS) -> dict:
    """Quantise the residual rows of one encode call, given in slot order.

    EK, EV: fp32 [H][n][128].  Keys: one group per (64 consecutive slots,
    channel); the last group holds only the rows present.  Values: one group per
    (row, 64-channel half).  Returns kc/vc uint8 [H][n][128], ks/kz fp16
    [H][ceil(n/64)][128], vs/vz fp16 [H][n][2].  ``levels`` 3 gives 2-bit codes.
    """
    EK = np.asarray(EK, F32)
    EV = np.asarray(EV, F32)
    H, n, D = EK.shape
    ng = -(-n // GROUP)
    kc = np.zeros((H, n, D), np.uint8)
    ks = np.zeros((H, ng, D), F16)
    kz = np.zeros((H, ng, D), F16)
    for g in range(ng):
        sl = slice(g * GROUP, min(n, (g + 1) * GROUP))
        kc[:, sl], ks[:, g], kz[:, g] = quantize(EK[:, sl, :], axis=1, levels=levels)
    vc, vs, vz = quantize(EV.reshape(H, n, 2, D // 2), axis=3, levels=levels)
    return dict(kc=kc, ks=ks, kz=kz, vc=vc.reshape(H, n, D), vs=vs, vz=vz)


def decode_residual(enc: dict):
    """Dequantised residual rows (EK_hat, EV_hat) fp32 [H][n][128]."""
    H, n, D = enc["kc"].shape
    kh = np.zeros((H, n, D), F32)
    for g in range(enc["ks"].shape[1]):
        sl = slice(g * GROUP, min(n, (g + 1) * GROUP))
        kh[:, sl] = dequant(enc["kc"][:, sl], enc["ks"][:, g][:, None, :], enc["kz"][:, g][:, None, :])
    vh = dequant(enc["vc"].reshape(H, n, 2, D // 2), enc["vs"][..., None],
                 enc["vz"][..., None]).reshape(H, n, D)
    return kh, vh


# ----------------------------------------------------------------------------
# Attention  ([Project] Step 02; [Guide] section 3 "Loop-aware sparse attention")
# ----------------------------------------------------------------------------
def softmax(l, axis=-1):
    l = np.asarray(l, F64)
    e = np.exp(l - l.max(axis=axis, keepdims=True))
    return e / e.sum(axis=axis, keepdims=True)


def logits(q, Kc) -> np.ndarray:
    """l_j = q . k_j / sqrt(128) in fp64.  q [H][128], Kc [H][N][128] -> [H][N]."""
    return np.einsum("hnd,hd->hn", np.asarray(Kc, F64), np.asarray(q, F64)) / np.sqrt(F64(HEAD_DIM))


def attention_dense(q, Kc, Vc):
    """Single-query attention over all N columns, no mask (the query is the last token).

    Returns (o [H][128], p [H][N], l [H][N]), all fp64.
    """
    l = logits(q, Kc)
    p = softmax(l)
    o = np.einsum("hn,hnd->hd", p, np.asarray(Vc, F64))
    return o, p, l


def select_topk(p_tilde, k: int) -> np.ndarray:
    """S: the k columns of largest p_tilde per head (ties to the smaller index), ascending.

    p_tilde [H][N] -> int64 [H][k].
    """
    p_tilde = np.asarray(p_tilde, F64)
    H, N = p_tilde.shape
    assert 1 <= k <= N
    out = np.empty((H, k), np.int64)
    idx = np.arange(N)
    for h in range(H):
        order = np.lexsort((idx, -p_tilde[h]))
        out[h] = np.sort(order[:k])
    return out


def selected_mass(p_tilde, S) -> np.ndarray:
    """m = sum over S of p_tilde: the selected columns' share of the preceding distribution."""
    return np.take_along_axis(np.asarray(p_tilde, F64), S, axis=1).sum(axis=1)


def unselected_contribution(p_tilde, lam, v_at_loop, S) -> np.ndarray:
    """u = sum over j not in S of p_tilde_j * v_hat_j at loop lam_j.

    ``v_at_loop(r)`` returns the fp32 values [H][N][128] every column has in loop r.
    """
    p_tilde = np.asarray(p_tilde, F64)
    H, N = p_tilde.shape
    keep = np.ones((H, N), bool)
    np.put_along_axis(keep, S, False, axis=1)
    u = np.zeros((H, HEAD_DIM), F64)
    for r in np.unique(lam):
        w = np.where(keep & (lam == r), p_tilde, 0.0)
        u += np.einsum("hn,hnd->hd", w, np.asarray(v_at_loop(int(r)), F64))
    return u


def attention_sparse(q, Kc, Vc, S, m, u):
    """o = u + m * softmax_S(q K_S^T / sqrt(d)) V_S.

    Returns (o [H][128], pi [H][k], l_S [H][k]), fp64; pi is the softmax over S.
    """
    KS = np.take_along_axis(np.asarray(Kc, F64), S[:, :, None], axis=1)
    VS = np.take_along_axis(np.asarray(Vc, F64), S[:, :, None], axis=1)
    lS = logits(q, KS)
    pi = softmax(lS)
    o = np.asarray(u, F64) + np.asarray(m, F64)[:, None] * np.einsum("hk,hkd->hd", pi, VS)
    return o, pi, lS


# ----------------------------------------------------------------------------
# Cross-loop token-sparse updates  ([Project] "The Method", Step 01: only the
# tokens that stay active are updated; [Guide] section 3 "Cross-loop token-sparse
# updates": after the dense early loops each loop ranks the previously updated
# tokens by normalized hidden-state change, keeps a top-k subset, and later
# selections are restricted to earlier active sets, so the sets nest)
# ----------------------------------------------------------------------------
def token_change(h_prev, h_cur) -> np.ndarray:
    """Squared normalized hidden-state change of each token row, fp64:

        key_j = ||h_cur[j] - h_prev[j]||^2 / ||h_prev[j]||^2

    (delta_j^2; ranking by it is ranking by delta_j).  BF16 inputs widen exactly to
    fp64.  A row whose previous state is all zero has key +inf when it changed and 0
    when it did not.
    """
    hp = np.asarray(h_prev, F64)
    hc = np.asarray(h_cur, F64)
    num = np.sum((hc - hp) ** 2, axis=-1)
    den = np.sum(hp ** 2, axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        key = num / den
    return np.where((den == 0) & (num == 0), 0.0, key)


def select_active(h_prev, h_cur, prev_rows, k: int) -> np.ndarray:
    """A_r from A_{r-1}: the k tokens of ``prev_rows`` (those updated in loop r-1)
    whose hidden state changed most in loop r-1, measured by ``token_change`` of
    their states entering (h_prev = h^(r-2)) and leaving (h_cur = h^(r-1)) that
    loop; ties go to the lower token; returned in ascending token order (int64).
    """
    prev_rows = np.asarray(prev_rows, np.int64)
    assert 0 <= k <= prev_rows.size
    key = token_change(np.asarray(h_prev)[prev_rows], np.asarray(h_cur)[prev_rows])
    order = np.lexsort((prev_rows, -key))
    return np.sort(prev_rows[order[:k]])


def nested_active_sets(h, n_active) -> list:
    """A_1 .. A_R from hidden states h[0..R-1] (h[0] enters loop 1, h[r] leaves loop r)
    and the per-loop sizes n_active[r]: A_1 is every token; a loop whose size is not
    smaller than its predecessor's keeps that set; otherwise A_r = select_active(
    h[r-2], h[r-1], A_{r-1}, n_active[r]).  Entry 0 of the result is None.
    """
    n = np.asarray(h[0]).shape[0]
    sets = [None, np.arange(n, dtype=np.int64)]
    for r in range(2, len(n_active)):
        prev = sets[r - 1]
        k = min(int(n_active[r]), prev.size)
        sets.append(prev.copy() if k == prev.size else select_active(h[r - 2], h[r - 1], prev, k))
    return sets


# ----------------------------------------------------------------------------
# Sparse prefill attention  ([Project] "The Method", Step 01: in a token-sparse
# loop only the active tokens are recomputed; the paragraph after Step 03: the
# selected tokens are gathered into compact buffers so that the work stays a regular
# GEMM)
# ----------------------------------------------------------------------------
def prefill_attention(q_act, pos, K, V) -> np.ndarray:
    """Causal attention of the active tokens of one loop, fp64.

    q_act [H][n_act][D]: the queries of the active tokens (compact, in token order);
    pos [n_act]: their token positions (ascending); K, V [H][N][D]: every token's key
    and value in this loop (an active token's new ones, an inactive token's reused
    from the previous loop).  Row i attends over the keys 0..pos[i] with scale
    1/sqrt(D); returns o [H][n_act][D].
    """
    q = np.asarray(q_act, F64)
    K = np.asarray(K, F64)
    V = np.asarray(V, F64)
    pos = np.asarray(pos, np.int64)
    H, n, D = q.shape
    o = np.zeros((H, n, D), F64)
    for i in range(n):
        j = int(pos[i]) + 1
        l = np.einsum("hd,hnd->hn", q[:, i], K[:, :j]) / np.sqrt(D)
        p = softmax(l)
        o[:, i] = np.einsum("hn,hnd->hd", p, V[:, :j])
    return o


# ----------------------------------------------------------------------------
# One layer's cross-loop cache and decode state
# ----------------------------------------------------------------------------
class OracleLayer:
    """The cross-loop cache of one layer for H heads, kept in logical form.

    Holds the base codes, one list of encode calls per residual loop, the fp32
    reconstructions X_hat^(r) of every quantised token, the BF16 tail of every
    loop, and the attention state (p_tilde, lam) the sparse loops need.
    """

    def __init__(self, heads: int, loops: int, capacity: int, codec: int = RESIDUAL_INT4):
        assert codec in (RESIDUAL_INT4, FULL_INT4, RESIDUAL_INT2)
        self.H, self.R, self.cap, self.codec = heads, loops, capacity, codec
        D = HEAD_DIM
        self.n_q = 0
        self.n_tail = 0
        self.base = dict(
            kc=np.zeros((heads, capacity, D), np.uint8), vc=np.zeros((heads, capacity, D), np.uint8),
            ks=np.zeros((heads, capacity // GROUP, D), F16), kz=np.zeros((heads, capacity // GROUP, D), F16),
            vs=np.zeros((heads, capacity, 2), F16), vz=np.zeros((heads, capacity, 2), F16))
        self.calls = {r: [] for r in range(2, loops + 1)}
        self.khat = np.zeros((loops + 1, heads, capacity, D), F32)
        self.vhat = np.zeros((loops + 1, heads, capacity, D), F32)
        self.depth = np.zeros(capacity, np.uint8)
        self.tail_k = np.zeros((loops + 1, heads, TAIL, D), F32)
        self.tail_v = np.zeros((loops + 1, heads, TAIL, D), F32)
        self.tail_depth = np.zeros(TAIL, np.uint8)
        self.p_tilde = None
        self.lam = None

    # -- encoders ------------------------------------------------------------
    def encode_base(self, row0: int, K1, V1):
        """Loop-1 base of tokens [row0, row0 + T)."""
        T = K1.shape[1]
        assert row0 % GROUP == 0 and T % GROUP == 0 and row0 + T <= self.cap
        enc = encode_base(K1, V1)
        sl = slice(row0, row0 + T)
        for key in ("kc", "vc", "vs", "vz"):
            self.base[key][:, sl] = enc[key]
        bl = slice(row0 // GROUP, (row0 + T) // GROUP)
        self.base["ks"][:, bl] = enc["ks"]
        self.base["kz"][:, bl] = enc["kz"]
        kh, vh = decode_base(enc)
        for r in range(1, self.R + 1):
            self.khat[r][:, sl] = kh
            self.vhat[r][:, sl] = vh
        self.depth[sl] = 1
        self.n_q = max(self.n_q, row0 + T)
        return enc

    def encode_residual(self, r: int, rows, Kr, Vr):
        """Loop-r store of the active ``rows`` (ascending token ids) of one call.

        Kr, Vr: fp32 [H][n][128], the loop-r keys/values of those rows.  The
        residual is taken against the reconstructed state of loop r-1 and added back
        onto it; with the per-loop KIVI4 codec the store holds the state itself and
        replaces the earlier reconstruction.
        """
        rows = np.asarray(rows, np.int64)
        assert 2 <= r <= self.R
        if rows.size:
            assert np.all(np.diff(rows) > 0) and rows[-1] < self.n_q
            assert np.all(self.depth[rows] >= r - 1), "active sets must nest"
        if self.codec == FULL_INT4:
            enc = encode_residual(np.asarray(Kr, F32), np.asarray(Vr, F32))
            newk, newv = decode_residual(enc)
        else:
            prev_k = self.khat[r - 1][:, rows]
            prev_v = self.vhat[r - 1][:, rows]
            EK = np.subtract(np.asarray(Kr, F32), prev_k, dtype=F32)
            EV = np.subtract(np.asarray(Vr, F32), prev_v, dtype=F32)
            enc = encode_residual(EK, EV, LEVELS2 if self.codec == RESIDUAL_INT2 else LEVELS)
            dk, dv = decode_residual(enc)
            newk = np.add(prev_k, dk, dtype=F32)
            newv = np.add(prev_v, dv, dtype=F32)
        for rr in range(r, self.R + 1):
            self.khat[rr][:, rows] = newk
            self.vhat[rr][:, rows] = newv
        self.depth[rows] = r
        self.calls[r].append(dict(rows=rows, enc=enc))
        return enc

    # -- tail ----------------------------------------------------------------
    def set_tail(self, Kt, Vt, depth):
        """Prompt tail: Kt/Vt indexed [r][H][t][128] for r = 1..R, depth [t]."""
        t = Kt[1].shape[1]
        assert 1 <= t <= TAIL
        for r in range(1, self.R + 1):
            self.tail_k[r][:, :t] = Kt[r]
            self.tail_v[r][:, :t] = Vt[r]
        self.tail_depth[:t] = depth
        self.n_tail = t

    def flush_tail(self):
        """Encode the 64 tail rows into the base and the residual stores."""
        assert self.n_tail == TAIL
        row0 = self.n_q
        self.encode_base(row0, self.tail_k[1], self.tail_v[1])
        for r in range(2, self.R + 1):
            idx = np.nonzero(self.tail_depth >= r)[0]
            self.encode_residual(r, row0 + idx, self.tail_k[r][:, idx], self.tail_v[r][:, idx])
        self.n_tail = 0

    def append_token(self, k, v):
        """Add the newest token (active in every loop): k/v indexed [r][H][128]."""
        if self.n_tail == TAIL:
            self.flush_tail()
        t = self.n_tail
        for r in range(1, self.R + 1):
            self.tail_k[r][:, t] = k[r]
            self.tail_v[r][:, t] = v[r]
        self.tail_depth[t] = self.R
        self.n_tail = t + 1

    @property
    def n_cols(self) -> int:
        return self.n_q + self.n_tail

    def columns(self, r: int):
        """(K, V) of every column in loop r: fp32 [H][N][128]."""
        k = np.concatenate([self.khat[r][:, :self.n_q], self.tail_k[r][:, :self.n_tail]], axis=1)
        v = np.concatenate([self.vhat[r][:, :self.n_q], self.tail_v[r][:, :self.n_tail]], axis=1)
        return k, v

    # -- decode loops ----------------------------------------------------------
    def dense_loop(self, r: int, q):
        """Full attention of loop r; p_tilde becomes its distribution, lam = r."""
        Kc, Vc = self.columns(r)
        o, p, l = attention_dense(q, Kc, Vc)
        self.p_tilde = p
        self.lam = np.full(p.shape, r, np.int64)
        return dict(o=o, p=p, l=l)

    def select(self, k: int):
        """The oracle's own (S, m, u) for the next sparse loop."""
        S = select_topk(self.p_tilde, k)
        return S, selected_mass(self.p_tilde, S), self.unselected(S)

    def unselected(self, S):
        return unselected_contribution(self.p_tilde, self.lam, lambda r: self.columns(r)[1], S)

    def sparse_loop(self, r: int, q, S):
        """Sparse attention of loop r over the columns S, then splice p_tilde and lam."""
        S = np.asarray(S, np.int64)
        m = selected_mass(self.p_tilde, S)
        u = self.unselected(S)
        Kc, Vc = self.columns(r)
        o, pi, lS = attention_sparse(q, Kc, Vc, S, m, u)
        np.put_along_axis(self.p_tilde, S, m[:, None] * pi, axis=1)
        np.put_along_axis(self.lam, S, r, axis=1)
        return dict(o=o, m=m, u=u, pi=pi, l=lS, S=S)

    def output_identity(self):
        """sum_j p_tilde_j * v_hat_j at loop lam_j: equals the last loop's output."""
        return unselected_contribution(self.p_tilde, self.lam, lambda r: self.columns(r)[1],
                                       np.zeros((self.H, 0), np.int64))

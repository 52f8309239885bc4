"""Seeded synthetic FlashLoop workloads.

The pages evaluate on trained Ouro/Huginn checkpoints and public benchmarks that
are not available here; these generators stand in for them with Gaussian data
of the same shapes:

* loop-1 keys/values are BF16-rounded N(0,1) draws;
* loop r >= 2 changes only its active rows, by BF16(previous + sigma_r * N(0,1)),
  and inactive rows keep the previous loop's state (project page, The Method,
  Step 01: inactive tokens reuse the preceding loop's KV);
* active sets are nested random subsets, drawn per token and shared by every
  layer and head (flozi guide "FlashLoop: store changes between repeated
  passes", section 3: later selections are restricted to earlier active sets);
* queries are BF16-rounded N(0,1) draws, independent per (layer, step, loop).

Nothing here quantises, reconstructs or attends: the method's arithmetic lives
in ``oracle/`` (reference side) and in the CUDA library (product side), which
both consume these tensors byte for byte.
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass

import torch

HEAD_DIM = 128
GROUP = 64
TAIL = 64


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: cache shape, loop schedule and seeds."""

    name: str
    layers: int
    heads: int
    n_ctx: int              # columns at the end of prefill (quantised + tail)
    loops: int              # R
    sigma: tuple            # sigma[r], r = 0..R (entries 0 and 1 unused)
    frac: tuple             # active fraction of loop r, r = 0..R (entry 0 unused)
    seed: int
    decode_steps: int = 0
    dense_loops: int = 2
    key_pct: int = 10       # retained key columns in sparse loops, percent

    def n_active(self, r: int, n_tokens: int) -> int:
        """|A_r| = ceil(frac_r * n) (exact for the 25 % / 10 % schedule)."""
        f = self.frac[r]
        if f >= 1.0:
            return n_tokens
        return min(n_tokens, math.ceil(f * n_tokens - 1e-9))

    def k_sel(self, n_cols: int) -> int:
        """ceil(key_pct / 100 * N) in integer arithmetic."""
        return (n_cols * self.key_pct + 99) // 100

    def layer_seed(self, layer: int) -> int:
        return self.seed + layer


def _four_loop(seed, name, layers, heads, n_ctx, decode_steps=0):
    return Workload(
        name=name, layers=layers, heads=heads, n_ctx=n_ctx, loops=4,
        sigma=(0.0, 0.0, 0.5, 0.2, 0.1), frac=(0.0, 1.0, 1.0, 0.25, 0.10),
        seed=seed, decode_steps=decode_steps)


def _deep(seed, name, heads, n_ctx, loops=32):
    sig = tuple([0.0, 0.0] + [0.5 * 0.85 ** r for r in range(2, loops + 1)])
    frac = tuple([0.0] + [0.05 ** ((r - 1) / (loops - 1)) for r in range(1, loops + 1)])
    return Workload(name=name, layers=1, heads=heads, n_ctx=n_ctx, loops=loops,
                    sigma=sig, frac=frac, seed=seed)


WORKLOADS = {
    w.name: w for w in (
        _four_loop(1000, "tiny_h1_n256", 1, 1, 256),
        _four_loop(1001, "layer_h16_n4096", 1, 16, 4096),
        _four_loop(1002, "layer_h16_n32768_decode256", 1, 16, 32768, decode_steps=256),
        _four_loop(3000, "cache_l48_h16_n32768", 48, 16, 32768),
        _deep(1004, "deep_r32_h16_n8192", 16, 8192),
    )
}


def split_prefill(n_cols: int) -> tuple[int, int]:
    """(n_q, n_tail): quantised tokens (a multiple of 64) and BF16 tail rows in [1, 64]."""
    if n_cols < 1:
        raise ValueError("need at least one column")
    n_tail = n_cols - GROUP * ((n_cols - 1) // GROUP)
    return n_cols - n_tail, n_tail


def _generator(device, *key) -> torch.Generator:
    h = hashlib.blake2b(repr(key).encode(), digest_size=8).digest()
    g = torch.Generator(device=device)
    g.manual_seed(int.from_bytes(h, "little") & ((1 << 63) - 1))
    return g


def _bf16_normal(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def active_sets(w: Workload, n_tokens: int) -> list:
    """Nested active sets A_1 ⊇ A_2 ⊇ ... ⊇ A_R over tokens [0, n_tokens).

    Returns a list indexed by loop r (entry 0 is None); each entry is a sorted
    int64 CPU tensor of token indices.
    """
    g = _generator("cpu", "active", w.seed, n_tokens)
    sets = [None, torch.arange(n_tokens, dtype=torch.int64)]
    for r in range(2, w.loops + 1):
        prev = sets[r - 1]
        k = min(w.n_active(r, n_tokens), prev.numel())
        if k == prev.numel():
            sets.append(prev.clone())
            continue
        pick = torch.randperm(prev.numel(), generator=g)[:k]
        sets.append(torch.sort(prev[pick]).values)
    return sets


def depth_of(sets: list, n_tokens: int) -> torch.Tensor:
    """D_j = max{r : j in A_r} as uint8 (1 for tokens active only in loop 1)."""
    d = torch.zeros(n_tokens, dtype=torch.uint8)
    for r in range(1, len(sets)):
        d[sets[r]] = r
    return d


def prefill_layer(w: Workload, layer: int, device="cpu", sets=None) -> dict:
    """Per-loop keys and values of every prompt token of one layer.

    Returns {"K": [None, K1..KR], "V": [...], "sets": sets}; each K[r] / V[r] is a
    BF16 tensor [H][n_ctx][128] on ``device``.
    """
    n = w.n_ctx
    if sets is None:
        sets = active_sets(w, n)
    g = _generator(device, "prefill", w.layer_seed(layer))
    shape = (w.heads, n, HEAD_DIM)
    K = [None, _bf16_normal(shape, g, device)]
    V = [None, _bf16_normal(shape, g, device)]
    for r in range(2, w.loops + 1):
        nk = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        nv = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        a = sets[r].to(device)
        kr, vr = K[r - 1].clone(), V[r - 1].clone()
        sig = float(w.sigma[r])
        kr[:, a] = (K[r - 1][:, a].float() + sig * nk[:, a]).to(torch.bfloat16)
        vr[:, a] = (V[r - 1][:, a].float() + sig * nv[:, a]).to(torch.bfloat16)
        K.append(kr)
        V.append(vr)
        del nk, nv
    return {"K": K, "V": V, "sets": sets}


def decode_token(w: Workload, layer: int, step: int, device="cpu") -> dict:
    """Per-loop key/value rows of the token generated at decode ``step``.

    A decode token is active in every loop. Returns {"k": [None, k1..kR],
    "v": [...]} with BF16 tensors [H][128].
    """
    g = _generator(device, "decode", w.layer_seed(layer), step)
    shape = (w.heads, HEAD_DIM)
    k = [None, _bf16_normal(shape, g, device)]
    v = [None, _bf16_normal(shape, g, device)]
    for r in range(2, w.loops + 1):
        nk = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        nv = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        sig = float(w.sigma[r])
        k.append((k[r - 1].float() + sig * nk).to(torch.bfloat16))
        v.append((v[r - 1].float() + sig * nv).to(torch.bfloat16))
    return {"k": k, "v": v}


def hidden_states(w: Workload, n_tokens: int, d_model: int, device="cpu", loops=None) -> list:
    """Hidden states for the token selector: h[0..R-1], BF16 [n_tokens][d_model].

    h[0] enters loop 1 and h[r] leaves loop r: h[0] = bf16(N(0,1)) and
    h[r] = bf16(h[r-1] + c_r g_{r,j} N(0,1)) with c_1 = 1, c_r = sigma_r for r >= 2 and
    a per-token magnitude g_{r,j} = exp(N(0,1)), so a few tokens move much more than the
    rest.  Every row is drawn as if its token were updated in every loop; a selector
    reads only the rows of the tokens it ranks.
    """
    R = w.loops if loops is None else loops
    g = _generator(device, "hidden", w.seed, n_tokens, d_model)
    h = [_bf16_normal((n_tokens, d_model), g, device)]
    for r in range(1, R):
        c = 1.0 if r == 1 else float(w.sigma[r])
        mag = torch.exp(torch.randn(n_tokens, generator=g, device=device, dtype=torch.float32))
        noise = torch.randn((n_tokens, d_model), generator=g, device=device, dtype=torch.float32)
        h.append((h[-1].float() + (c * mag)[:, None] * noise).to(torch.bfloat16))
        del noise
    return h


def queries(w: Workload, layer: int, step: int, device="cpu") -> torch.Tensor:
    """BF16 queries [R + 1][H][128] (row 0 unused) for one decode step of one layer."""
    g = _generator(device, "query", w.layer_seed(layer), step)
    q = _bf16_normal((w.loops + 1, w.heads, HEAD_DIM), g, device)
    q[0].zero_()
    return q

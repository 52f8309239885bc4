"""Nested active token sets from hidden states, on the GPU.

FlashLoop project page, "The Method", Step 01, and the flozi guide "FlashLoop: store
changes between repeated passes", section 3: after the dense early loops each loop
ranks the tokens updated in the previous loop by normalized hidden-state change and
keeps a top-k subset, so A_1 = every token and A_r is a subset of A_{r-1}.  Each
ranking is one fl_select_active call.
"""
from __future__ import annotations

import torch

from . import abi


def nested_active_sets(h, n_active, stream=None) -> list:
    """A_1 .. A_R as device int32 tensors (ascending); entry 0 is None.

    ``h[0..R-1]``: BF16 [n_tokens][d] hidden states on the GPU (h[0] enters loop 1, h[r]
    leaves loop r).  ``n_active[r]``: the size of A_r.  A loop not smaller than its
    predecessor keeps that set; otherwise A_r is the n_active[r] tokens of A_{r-1} whose
    state changed most over loop r-1 (h[r-2] -> h[r-1]).
    """
    n = h[0].shape[0]
    dev = h[0].device
    sets = [None, torch.arange(n, dtype=torch.int32, device=dev)]
    keys = torch.empty(n, dtype=torch.float64, device=dev)
    for r in range(2, len(n_active)):
        prev = sets[r - 1]
        k = min(int(n_active[r]), prev.numel())
        if k == prev.numel():
            sets.append(prev.clone())
            continue
        out = torch.empty(k, dtype=torch.int32, device=dev)
        abi.fl_select_active(h[r - 2], h[r - 1], prev, k, out, keys, stream=stream)
        sets.append(out)
    return sets

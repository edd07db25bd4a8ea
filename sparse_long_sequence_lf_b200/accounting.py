"""Work accounting for throughput and roofline figures (host arithmetic only).

Useful work counts the (query, key) pairs the method attends: for each valid
local row the size of (window taps UNION global tokens) INTERSECT valid
tokens; for each valid global row the number of valid tokens.  Padded rows,
taps outside the sequence and global keys already inside the window are not
counted.  Each pair costs 2*d flops for the score and 2*d for the weighted
value: FLOPs = 4 * d * pairs.  The complexity the pages state for the method
is O(n * (w + g)) ("Longformer模型深度解析与应用指南", core technique section).

Algorithmic bytes are what one forward must move at least once: Q, K, V and
the output in full, Kg and Vg in full when any global token exists, and the
Qg rows of the global tokens.
"""
from __future__ import annotations

import numpy as np

from .workloads import Workload, global_positions, make_masks

ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


def _masks_np(wl: Workload):
    local, glob = make_masks(wl)
    lm = np.ones((wl.B, wl.n), dtype=bool) if local is None else local.numpy() != 0
    gm = np.zeros((wl.B, wl.n), dtype=bool) if glob is None else glob.numpy() != 0
    return lm, gm


def _tap_counts(valid: np.ndarray, w: int, dil: int, causal: bool) -> np.ndarray:
    """Per row i: number of valid keys among its window taps (inside [0, n))."""
    n = valid.shape[0]
    cnt = np.zeros(n, dtype=np.int64)
    offs = range(0, -w, -1) if causal else range(-(w // 2), w // 2 + 1)
    idx = np.arange(n)
    for k in offs:
        j = idx + k * dil
        ok = (j >= 0) & (j < n)
        cnt[ok] += valid[j[ok]]
    return cnt


def _global_extra(valid, gpos, w, dil, causal) -> np.ndarray:
    """Per row i: valid global keys that are not window taps of i."""
    n = valid.shape[0]
    i = np.arange(n)
    extra = np.zeros(n, dtype=np.int64)
    for j in gpos:
        if not valid[j]:
            continue
        diff = j - i
        if causal:
            back = -diff
            tap = (back >= 0) & (back % dil == 0) & (back // dil <= w - 1)
        else:
            a = np.abs(diff)
            tap = (a % dil == 0) & (a // dil <= w // 2)
        extra += ~tap
    return extra


def useful_pairs(wl: Workload) -> int:
    lm, gm = _masks_np(wl)
    gpos_all = global_positions(wl)
    total = 0
    dils = wl.dilation_list()
    for b in range(wl.B):
        valid = lm[b]
        nvalid = int(valid.sum())
        is_g = gm[b]
        local_rows = valid & ~is_g
        n_global_rows = int((valid & is_g).sum())
        cache = {}
        for h in range(wl.H):
            d = dils[h]
            if d not in cache:
                per_row = _tap_counts(valid, wl.window, d, wl.causal)
                per_row = per_row + _global_extra(valid, gpos_all[b], wl.window, d, wl.causal)
                cache[d] = int(per_row[local_rows].sum())
            total += cache[d] + n_global_rows * nvalid
    return total


def useful_flops(wl: Workload) -> int:
    return 4 * wl.d * useful_pairs(wl)


def useful_flops_rows(wl: Workload, head: int, rows: tuple, batch: int = 0) -> int:
    """FLOPs of the attended pairs of rows [rows[0], rows[1]) of one (batch,
    head): the same count as useful_flops, restricted to those rows."""
    lm, gm = _masks_np(wl)
    valid = lm[batch]
    d = wl.dilation_list()[head]
    per_row = _tap_counts(valid, wl.window, d, wl.causal)
    per_row = per_row + _global_extra(valid, global_positions(wl)[batch], wl.window, d, wl.causal)
    sel = np.zeros(wl.n, dtype=bool)
    sel[rows[0]:rows[1]] = True
    local_rows = sel & valid & ~gm[batch]
    global_rows = sel & valid & gm[batch]
    pairs = int(per_row[local_rows].sum()) + int(global_rows.sum()) * int(valid.sum())
    return 4 * wl.d * pairs


def algorithmic_bytes(wl: Workload) -> int:
    e = ELEM_BYTES[wl.dtype]
    full = wl.B * wl.H * wl.n * wl.d * e
    g_rows = sum(len(p) for p in global_positions(wl))
    total = 4 * full                                  # Q, K, V, O
    if g_rows > 0:
        total += 2 * full                             # Kg, Vg
        total += wl.H * g_rows * wl.d * e             # Qg at the global rows
    return total


def tokens(wl: Workload) -> int:
    return wl.B * wl.n


def backward_flops(wl: Workload) -> int:
    """FLOPs of one backward over the same pairs: five products of 2*d flops
    per pair (the recomputed score, dP = dO.v, and the dq, dk, dv sums)."""
    return 10 * wl.d * useful_pairs(wl)


# CUDA-core fp32 peak of a B200: 148 SMs x 128 fp32 lanes x 2 flops (FMA)
# per clock; multiplied by the SM clock in MHz it gives MFLOP/s.
FP32_FLOPS_PER_CLOCK = 148 * 128 * 2

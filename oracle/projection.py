"""fp64 oracle of the projection prologue of the Longformer attention.

TEST INFRASTRUCTURE ONLY: the test suite and the benchmark's CPU-baseline leg
are the only callers.  The product library never imports or executes
anything in this directory, and this module imports nothing from the product
package.

What it computes (FasterTransformer Longformer Encoder guide, "compute
flow"): the hidden states X [B, n, H*d] of a layer are multiplied by five
weight matrices, each plus a bias, giving Q, K, V for the sliding window and
Kg, Vg for the global attention over every token; the global query Qg is the
same product with its own weights for the global tokens only (a batched
product over the gathered global rows).  Each product is then split into
heads and laid out [B, H, n, d] (the guide's bias-add-and-transpose step).
Here the definition is written out directly in fp64: y = W x + b per token,
with W stored as [out_features, in_features] (row o holds the weights of
output feature o), feature o = h*d + e of a projection going to head h,
dimension e.

Reading taken where the guide is silent: rows of Qg at positions that are
not global tokens are left as they were (the attention never reads them).
"""
from __future__ import annotations

import numpy as np

PROJECTIONS = ("q", "k", "v", "kg", "vg")   # order of the blocks of the stacked weights


def split_heads(y: np.ndarray, H: int, d: int) -> np.ndarray:
    """[B, n, H*d] -> [B, H, n, d]."""
    B, n, _ = y.shape
    return y.reshape(B, n, H, d).transpose(0, 2, 1, 3)


def projection_forward(x, w, bias, wqg, bqg, global_idx, counts, *, H: int, d: int = 64,
                       qg_init=None):
    """fp64 projections.

    x          [B, n, H*d] hidden states (values already rounded to the GPU's
               input dtype).
    w          [5*H*d, H*d] stacked weights of Q, K, V, Kg, Vg (rows = output
               features); bias [5*H*d] or None.
    wqg, bqg   [H*d, H*d] and [H*d] (or None): the global-query projection.
    global_idx [B, n] compacted global positions (ascending, -1 tail) and
    counts     [B]: which rows get Qg.
    qg_init    [B, H, n, d] values of Qg's non-global rows (default zeros).
    Returns a dict of [B, H, n, d] fp64 arrays for q, k, v, kg, vg, qg.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    B, n, hid = x.shape
    assert hid == H * d and w.shape == (5 * hid, hid)
    out = {}
    for p, name in enumerate(PROJECTIONS):
        wp = w[p * hid:(p + 1) * hid]                     # [hid_out, hid_in]
        y = np.einsum("bni,oi->bno", x, wp)
        if bias is not None:
            y = y + np.asarray(bias, dtype=np.float64)[p * hid:(p + 1) * hid]
        out[name] = split_heads(y, H, d)
    qg = (np.zeros((B, H, n, d)) if qg_init is None
          else np.array(qg_init, dtype=np.float64, copy=True))
    wqg = np.asarray(wqg, dtype=np.float64)
    for b in range(B):
        g = int(counts[b])
        rows = np.asarray(global_idx[b][:g], dtype=np.int64)
        if g == 0:
            continue
        y = x[b, rows] @ wqg.T                            # [g, hid]
        if bqg is not None:
            y = y + np.asarray(bqg, dtype=np.float64)
        qg[b][:, rows, :] = y.reshape(g, H, d).transpose(1, 0, 2)
    out["qg"] = qg
    return out


def output_layer(attn, wo, bo, residual, gamma, beta, *, eps: float = 1e-5):
    """fp64 output layer of the attention block (FasterTransformer Longformer
    Encoder guide, "compute flow": the heads are concatenated back into one
    [B, n, H*d] tensor, multiplied by the output weight matrix plus bias, the
    layer input is added back and the sum layer-normalised with its own
    scale and shift).

    attn     [B, H, n, d] attention output.
    wo, bo   [H*d, H*d] (rows = output features) and [H*d] or None.
    residual [B, n, H*d] the layer input.
    gamma, beta [H*d]; eps added to the variance (the population variance
    over the H*d features of a token).
    Returns [B, n, H*d] fp64.
    """
    a = np.asarray(attn, dtype=np.float64)
    B, H, n, d = a.shape
    merged = a.transpose(0, 2, 1, 3).reshape(B, n, H * d)
    y = np.einsum("bni,oi->bno", merged, np.asarray(wo, dtype=np.float64))
    if bo is not None:
        y = y + np.asarray(bo, dtype=np.float64)
    y = y + np.asarray(residual, dtype=np.float64)
    mean = y.mean(axis=-1, keepdims=True)
    var = ((y - mean) ** 2).mean(axis=-1, keepdims=True)
    z = (y - mean) / np.sqrt(var + eps)
    return z * np.asarray(gamma, dtype=np.float64) + np.asarray(beta, dtype=np.float64)

"""fp64 oracle of the backward pass of the Longformer self-attention.

TEST INFRASTRUCTURE ONLY: the test suite and the benchmark's CPU-baseline leg
are the only callers.  The product library never imports or executes
anything in this directory, and this module imports nothing from the product
package.

What it differentiates: the forward of the same attention ("LongFormer: The
Long-Document Transformer" notes, "Sliding Window", "Dilated Sliding
Window", "Global Attention"; FasterTransformer Longformer Encoder guide,
"compute flow"), written here independently of the C oracle as dense masked
attention in torch fp64: for every batch and head a boolean matrix marks the
keys of each query row (window taps and global tokens for a valid non-global
row, every valid token for a valid global row, nothing for a padded row);
local rows use Q, K, V and global rows Qg, Kg, Vg; rows with no keys output
zero.  torch.autograd then gives the gradients of sum(O * dO) with respect to
the six projections.  Small problems only (n x n masks).
"""
from __future__ import annotations

import numpy as np
import torch


def _is_tap(i: int, j: int, w: int, dil: int, causal: bool) -> bool:
    diff = j - i
    if causal:
        if diff > 0:
            return False
        back = -diff
        return back % dil == 0 and back // dil <= w - 1
    a = abs(diff)
    return a % dil == 0 and a // dil <= w // 2


def key_masks(local_mask, global_mask, *, B, H, n, window, dilation, causal):
    """Boolean [B, H, n, n] masks: local[b,h,i,j] (key j of local row i) and
    glob[b,h,i,j] (key j of global row i)."""
    valid = (np.ones((B, n), bool) if local_mask is None
             else np.asarray(local_mask).astype(bool))
    isg = (np.zeros((B, n), bool) if global_mask is None
           else np.asarray(global_mask).astype(bool))
    dil = list(dilation) if dilation is not None else [1] * H
    local = np.zeros((B, H, n, n), bool)
    glob = np.zeros((B, H, n, n), bool)
    for b in range(B):
        gpos = [j for j in range(n) if isg[b, j]]
        for h in range(H):
            for i in range(n):
                if not valid[b, i]:
                    continue
                if isg[b, i]:
                    glob[b, h, i] = valid[b]
                    continue
                for j in range(n):
                    if _is_tap(i, j, window, dil[h], causal):
                        local[b, h, i, j] = True
                for j in gpos:
                    local[b, h, i, j] = True
                local[b, h, i] &= valid[b]
    return local, glob


def _masked_attention(q, k, v, mask, scale):
    s = torch.einsum("bhid,bhjd->bhij", q, k) * scale
    s = s.masked_fill(~mask, float("-inf"))
    has = mask.any(dim=-1, keepdim=True)
    p = torch.softmax(torch.where(has, s, torch.zeros_like(s)), dim=-1)
    p = torch.where(mask, p, torch.zeros_like(p))
    return torch.einsum("bhij,bhjd->bhid", p, v)


def forward(q, k, v, qg, kg, vg, local_mask, global_mask, *, window, dilation=None,
            causal=False):
    """The forward of this oracle (fp64 tensors in, fp64 out)."""
    B, H, n, d = q.shape
    local, glob = key_masks(local_mask, global_mask, B=B, H=H, n=n, window=window,
                            dilation=dilation, causal=causal)
    lm, gm = torch.from_numpy(local), torch.from_numpy(glob)
    scale = 1.0 / np.sqrt(d)
    o_local = _masked_attention(q, k, v, lm, scale)
    o_glob = _masked_attention(qg, kg, vg, gm, scale)
    grow = gm.any(dim=-1, keepdim=True)
    return torch.where(grow, o_glob, o_local)


def backward(q, k, v, qg, kg, vg, local_mask, global_mask, dout, *, window, dilation=None,
             causal=False):
    """Gradients of sum(O * dout) as a dict of fp64 numpy arrays [B, H, n, d]
    for q, k, v, qg, kg, vg.  Inputs: arrays or tensors (any float type; the
    values are taken exactly)."""
    t = lambda a: torch.as_tensor(np.asarray(a, dtype=np.float64) if not torch.is_tensor(a)
                                  else a.double().numpy()).clone().requires_grad_(True)
    xs = [t(a) for a in (q, k, v, qg, kg, vg)]
    o = forward(*xs, local_mask, global_mask, window=window, dilation=dilation, causal=causal)
    g = torch.as_tensor(np.asarray(dout, dtype=np.float64) if not torch.is_tensor(dout)
                        else dout.double().numpy())
    (o * g).sum().backward()
    names = ("q", "k", "v", "qg", "kg", "vg")
    return {nm: x.grad.numpy() for nm, x in zip(names, xs)}

"""fp64 oracle of a whole Longformer encoder layer and of a stack of them.

TEST INFRASTRUCTURE ONLY: the test suite and the benchmark's CPU-baseline leg
are the only callers.  The product library never imports or executes
anything in this directory, and this module imports nothing from the product
package.

What one layer computes (FasterTransformer Longformer Encoder guide, "compute
flow", the per-layer loop):
  1. the projections Q, K, V, Kg, Vg of every token and Qg of the global
     tokens, each plus its bias, split into heads (projection.py);
  2. the Longformer attention over them (the C oracle, lf_oracle.c);
  3. heads concatenated, output weights plus bias, the layer input added
     back, LayerNorm (projection.output_layer);
  4. the feed-forward block: intermediate product plus bias, GELU, output
     product plus bias, the block input (the result of 3) added back, a
     second LayerNorm.
A stack applies the layers in order; each layer may have its own window and
dilations ("LongFormer: The Long-Document Transformer" notes, "Sliding
Window": a different w per layer; smaller windows low in the stack, larger
ones higher up).  The benchmark table of the same guide fixes the model it
times: 16 heads of 64, intermediate size 4096, window 512, 24 layers.

Readings taken where the pages are silent:
  * GELU is the exact form x * Phi(x) = x/2 * (1 + erf(x / sqrt 2)), not the
    tanh approximation (the pages name GELU only).
  * Both LayerNorms use the population variance over the features and the
    same eps.
  * A stack hands each layer's output to the next in the input dtype: the
    optional ``round_to`` rounds every layer output to it, because the
    layers' interface tensors are stored in that dtype.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

import oracle
from oracle.projection import output_layer, projection_forward

LAYER_KEYS = ("w_qkv", "b_qkv", "w_qg", "b_qg", "w_o", "b_o", "ln1_gamma", "ln1_beta",
              "w_1", "b_1", "w_2", "b_2", "ln2_gamma", "ln2_beta")


def gelu(x):
    """x * Phi(x), Phi the standard normal CDF written through erf."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def layer_norm(y, gamma, beta, eps):
    y = np.asarray(y, dtype=np.float64)
    mean = y.mean(axis=-1, keepdims=True)
    var = ((y - mean) ** 2).mean(axis=-1, keepdims=True)
    return (y - mean) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) \
        + np.asarray(beta, np.float64)


def ffn_block(h, w1, b1, w2, b2, gamma, beta, *, eps=1e-5):
    """LayerNorm(GELU(h W1^T + b1) W2^T + b2 + h).  h [B, n, hid];
    w1 [inter, hid], w2 [hid, inter] (rows = output features)."""
    h = np.asarray(h, dtype=np.float64)
    a = np.einsum("bni,oi->bno", h, np.asarray(w1, np.float64))
    if b1 is not None:
        a = a + np.asarray(b1, np.float64)
    a = gelu(a)
    y = np.einsum("bni,oi->bno", a, np.asarray(w2, np.float64))
    if b2 is not None:
        y = y + np.asarray(b2, np.float64)
    return layer_norm(y + h, gamma, beta, eps)


def _f64(t):
    if hasattr(t, "detach"):
        import torch
        return t.detach().to("cpu", torch.float64).numpy()
    return None if t is None else np.asarray(t, dtype=np.float64)


def encoder_layer(x, weights: dict, local_mask=None, global_mask=None, *, H: int, window: int,
                  dilation=None, eps: float = 1e-5, d: int = 64):
    """One layer.  x [B, n, H*d]; weights holds the LAYER_KEYS arrays
    (biases may be None; w_qg may be None when there are no global tokens).
    Returns (layer output, dict of the intermediate results)."""
    x = _f64(x)
    B, n, hid = x.shape
    w = {k: _f64(weights.get(k)) for k in LAYER_KEYS}
    if global_mask is not None:
        gidx, counts = oracle.global_index(global_mask)
    else:
        gidx, counts = np.full((B, n), -1, np.int32), np.zeros((B,), np.int32)
    wqg = w["w_qg"] if w["w_qg"] is not None else np.zeros((hid, hid))
    p = projection_forward(x, w["w_qkv"], w["b_qkv"], wqg, w["b_qg"], gidx, counts, H=H, d=d)
    attn = oracle.forward(p["q"], p["k"], p["v"], p["qg"], p["kg"], p["vg"], local_mask,
                          global_mask, window=window, dilation=dilation, causal=False)
    h1 = output_layer(attn, w["w_o"], w["b_o"], x, w["ln1_gamma"], w["ln1_beta"], eps=eps)
    out = ffn_block(h1, w["w_1"], w["b_1"], w["w_2"], w["b_2"], w["ln2_gamma"], w["ln2_beta"],
                    eps=eps)
    return out, {"proj": p, "attn": attn, "h1": h1}


def encoder_forward(x, layers, local_mask=None, global_mask=None, *, H: int, windows,
                    dilations=None, eps: float = 1e-5, round_to=None):
    """A stack: layer l with windows[l] and dilations[l] (a list of H values,
    or None for all 1).  round_to: a function applied to each layer's output
    before the next layer (the storage dtype of the layer interface)."""
    h = _f64(x)
    for l, wts in enumerate(layers):
        dil = None if dilations is None else dilations[l]
        h, _ = encoder_layer(h, wts, local_mask, global_mask, H=H, window=windows[l],
                             dilation=dil, eps=eps)
        if round_to is not None:
            h = round_to(h)
    return h

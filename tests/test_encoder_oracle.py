"""Pins of the encoder-layer oracle (oracle/encoder.py) against things other
than itself: the normal CDF of scipy.stats, closed-form identities of GELU,
torch's LayerNorm, and torch.nn.TransformerEncoderLayer in fp64, which is
what a Longformer layer reduces to when the window covers the whole sequence
(or every token is global) and nothing is padded."""
import numpy as np
import pytest
import torch
from scipy.stats import norm

from oracle import encoder as enc


def test_gelu_is_x_times_normal_cdf():
    x = np.linspace(-8, 8, 1001)
    assert np.allclose(enc.gelu(x), x * norm.cdf(x), rtol=0, atol=1e-14)
    assert enc.gelu(0.0) == 0.0
    # x Phi(x) - (-x) Phi(-x) = x, since Phi(x) + Phi(-x) = 1
    assert np.allclose(enc.gelu(x) - enc.gelu(-x), x, atol=1e-14)
    # Phi(1) = 0.841344746068543 (tabulated value of the standard normal CDF)
    assert abs(enc.gelu(1.0) - 0.841344746068543) < 1e-14


def test_layer_norm_matches_torch():
    rng = np.random.default_rng(1)
    y = rng.normal(size=(2, 5, 96)) * 3 + 1
    g, b = rng.normal(size=96), rng.normal(size=96)
    want = torch.nn.functional.layer_norm(torch.from_numpy(y), (96,), torch.from_numpy(g),
                                          torch.from_numpy(b), eps=1e-5).numpy()
    assert np.allclose(enc.layer_norm(y, g, b, 1e-5), want, atol=1e-12)


def _weights(rng, H, inter, d=64):
    hid = H * d
    s = 1 / np.sqrt(hid)
    return {
        "w_qkv": rng.normal(size=(5 * hid, hid)) * s, "b_qkv": rng.normal(size=5 * hid) * 0.1,
        "w_qg": rng.normal(size=(hid, hid)) * s, "b_qg": rng.normal(size=hid) * 0.1,
        "w_o": rng.normal(size=(hid, hid)) * s, "b_o": rng.normal(size=hid) * 0.1,
        "ln1_gamma": 1 + rng.normal(size=hid) * 0.1, "ln1_beta": rng.normal(size=hid) * 0.1,
        "w_1": rng.normal(size=(inter, hid)) * s, "b_1": rng.normal(size=inter) * 0.1,
        "w_2": rng.normal(size=(hid, inter)) / np.sqrt(inter), "b_2": rng.normal(size=hid) * 0.1,
        "ln2_gamma": 1 + rng.normal(size=hid) * 0.1, "ln2_beta": rng.normal(size=hid) * 0.1,
    }


def _torch_layer(w, H, inter, *, qkv_blocks=(0, 1, 2), eps=1e-5):
    """torch.nn.TransformerEncoderLayer (post-norm, exact GELU) holding the
    same weights; qkv_blocks picks which of the five stacked projections act
    as Q, K, V (0, 1, 2 the local ones; the global path uses Qg, 3, 4)."""
    hid = H * 64
    layer = torch.nn.TransformerEncoderLayer(hid, H, dim_feedforward=inter, dropout=0.0,
                                             activation="gelu", layer_norm_eps=eps,
                                             batch_first=True, norm_first=False,
                                             dtype=torch.float64)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    blocks_w, blocks_b = [], []
    for src in qkv_blocks:
        if src == "qg":
            blocks_w.append(w["w_qg"])
            blocks_b.append(w["b_qg"])
        else:
            blocks_w.append(w["w_qkv"][src * hid:(src + 1) * hid])
            blocks_b.append(w["b_qkv"][src * hid:(src + 1) * hid])
    with torch.no_grad():
        layer.self_attn.in_proj_weight.copy_(t(np.concatenate(blocks_w)))
        layer.self_attn.in_proj_bias.copy_(t(np.concatenate(blocks_b)))
        layer.self_attn.out_proj.weight.copy_(t(w["w_o"]))
        layer.self_attn.out_proj.bias.copy_(t(w["b_o"]))
        layer.linear1.weight.copy_(t(w["w_1"]))
        layer.linear1.bias.copy_(t(w["b_1"]))
        layer.linear2.weight.copy_(t(w["w_2"]))
        layer.linear2.bias.copy_(t(w["b_2"]))
        layer.norm1.weight.copy_(t(w["ln1_gamma"]))
        layer.norm1.bias.copy_(t(w["ln1_beta"]))
        layer.norm2.weight.copy_(t(w["ln2_gamma"]))
        layer.norm2.bias.copy_(t(w["ln2_beta"]))
    return layer.eval()


def test_full_window_layer_is_a_transformer_layer():
    rng = np.random.default_rng(2)
    H, n, inter = 2, 40, 256
    w = _weights(rng, H, inter)
    x = rng.normal(size=(2, n, H * 64))
    got, _ = enc.encoder_layer(x, w, H=H, window=2 * n)
    with torch.no_grad():
        want = _torch_layer(w, H, inter)(torch.from_numpy(x)).numpy()
    assert np.allclose(got, want, atol=1e-10)


def test_all_global_layer_uses_the_global_projections():
    rng = np.random.default_rng(3)
    H, n, inter = 2, 24, 128
    w = _weights(rng, H, inter)
    x = rng.normal(size=(1, n, H * 64))
    gm = np.ones((1, n), np.uint8)
    got, _ = enc.encoder_layer(x, w, None, gm, H=H, window=2)
    with torch.no_grad():
        want = _torch_layer(w, H, inter, qkv_blocks=("qg", 3, 4))(torch.from_numpy(x)).numpy()
    assert np.allclose(got, want, atol=1e-10)


def test_stack_applies_layers_in_order():
    rng = np.random.default_rng(4)
    H, n, inter = 1, 30, 128
    ws = [_weights(rng, H, inter) for _ in range(3)]
    x = rng.normal(size=(1, n, 64))
    got = enc.encoder_forward(x, ws, H=H, windows=[64, 80, 100])
    h = torch.from_numpy(x)
    with torch.no_grad():
        for w in ws:
            h = _torch_layer(w, H, inter)(h)
    assert np.allclose(got, h.numpy(), atol=1e-10)


def test_small_window_differs_from_full_attention():
    # A narrow window must change the result (the window actually masks).
    rng = np.random.default_rng(5)
    H, n, inter = 1, 64, 128
    w = _weights(rng, H, inter)
    x = rng.normal(size=(1, n, 64))
    narrow, _ = enc.encoder_layer(x, w, H=H, window=4)
    full, _ = enc.encoder_layer(x, w, H=H, window=2 * n)
    assert np.abs(narrow - full).max() > 1e-3
    # rows far from both ends see the same window under both windows only if
    # the window covers everything: check one explicit row by hand
    p = enc.encoder_layer(x, w, H=H, window=4)[1]["proj"]
    q, k, v = p["q"][0, 0], p["k"][0, 0], p["v"][0, 0]
    i = 30
    js = np.arange(i - 2, i + 3)
    s = q[i] @ k[js].T / 8.0
    pr = np.exp(s - s.max())
    pr /= pr.sum()
    attn = enc.encoder_layer(x, w, H=H, window=4)[1]["attn"][0, 0, i]
    assert np.allclose(attn, pr @ v[js], atol=1e-12)


def test_stack_gives_each_layer_its_own_window():
    # Layer 0 with a narrow window, layer 1 covering the sequence: the stack
    # equals that narrow layer followed by a full-attention transformer layer.
    rng = np.random.default_rng(6)
    H, n, inter = 1, 32, 128
    ws = [_weights(rng, H, inter) for _ in range(2)]
    x = rng.normal(size=(1, n, 64))
    got = enc.encoder_forward(x, ws, H=H, windows=[4, 2 * n])
    first, _ = enc.encoder_layer(x, ws[0], H=H, window=4)
    with torch.no_grad():
        want = _torch_layer(ws[1], H, inter)(torch.from_numpy(first)).numpy()
    assert np.allclose(got, want, atol=1e-10)


def test_padding_equals_truncation_through_the_stack():
    # Padded tokens are no keys of any row and every other step is per token,
    # so the valid rows of a padded sequence equal the stack on the truncated
    # sequence.
    rng = np.random.default_rng(7)
    H, n, t, inter = 1, 30, 6, 128
    ws = [_weights(rng, H, inter) for _ in range(2)]
    x = rng.normal(size=(1, n, 64))
    lm = np.ones((1, n), np.uint8)
    lm[0, n - t:] = 0
    gm = np.zeros((1, n), np.uint8)
    gm[0, 2] = 1
    got = enc.encoder_forward(x, ws, lm, gm, H=H, windows=[8, 8])
    want = enc.encoder_forward(x[:, :n - t], ws, None, gm[:, :n - t].copy(), H=H,
                               windows=[8, 8])
    assert np.allclose(got[:, :n - t], want, atol=1e-10)
    # and the padding does change the valid rows near the tail
    full = enc.encoder_forward(x, ws, None, gm, H=H, windows=[8, 8])
    assert np.abs(full[:, :n - t] - want).max() > 1e-6


def test_stack_gives_each_layer_its_own_dilations():
    rng = np.random.default_rng(8)
    H, n, inter = 2, 28, 128
    ws = [_weights(rng, H, inter) for _ in range(2)]
    x = rng.normal(size=(1, n, 128))
    dils = [[1, 2], [3, 1]]
    got = enc.encoder_forward(x, ws, H=H, windows=[6, 6], dilations=dils)
    h, _ = enc.encoder_layer(x, ws[0], H=H, window=6, dilation=dils[0])
    want, _ = enc.encoder_layer(h, ws[1], H=H, window=6, dilation=dils[1])
    assert np.allclose(got, want, atol=1e-12)
    other, _ = enc.encoder_layer(h, ws[1], H=H, window=6, dilation=dils[0])
    assert np.abs(other - want).max() > 1e-6

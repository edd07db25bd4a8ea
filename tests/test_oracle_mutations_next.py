"""Plant plausible mistakes in private copies of the backward and encoder
oracles and check that their pins catch every one (CPU only; the committed
oracles are untouched: each mutant is compiled into a fresh module)."""
import os
import types

import pytest

import test_backward_oracle as tb
import test_encoder_oracle as te
from oracle import backward as obw
from oracle import encoder as oenc


def _mutant(module, old, new):
    src = open(module.__file__).read()
    assert src.count(old) >= 1, f"mutation target not found: {old!r}"
    mod = types.ModuleType(module.__name__ + "_mutant")
    mod.__file__ = module.__file__
    exec(compile(src.replace(old, new), module.__file__, "exec"), mod.__dict__)
    return mod


def _caught(test_module, attr, mutant, calls):
    saved = getattr(test_module, attr)
    setattr(test_module, attr, mutant)
    caught = []
    try:
        for fn, args in calls:
            try:
                fn(*args)
            except Exception as e:              # a failed assertion or a crash
                caught.append((fn.__name__, type(e).__name__))
    finally:
        setattr(test_module, attr, saved)
    return caught


def _param_values(fn):
    return [m.args[1] for m in fn.pytestmark if m.name == "parametrize"][0]


BWD_PINS = ([(tb.test_forward_agrees_with_the_c_oracle, (kw,))
             for kw in _param_values(tb.test_forward_agrees_with_the_c_oracle)]
            + [(tb.test_gradients_agree_with_finite_differences_of_the_c_oracle, ()),
               (tb.test_padded_rows_and_unused_projections_get_no_gradient, ()),
               (tb.test_full_window_gradients_equal_sdpa_autograd, ()),
               (tb.test_all_global_gradients_equal_sdpa_autograd_on_global_projections, ())])

BWD_MUTATIONS = [
    ("window one tap short", "return a % dil == 0 and a // dil <= w // 2",
     "return a % dil == 0 and a // dil < w // 2"),
    ("dilation ignored (non-causal)", "return a % dil == 0 and a // dil <= w // 2",
     "return a <= w // 2"),
    ("causal looks right", "        if diff > 0:\n            return False",
     "        if diff < 0:\n            return False"),
    ("global keys dropped from local rows", "local[b, h, i, j] = True\n                local",
     "pass\n                local"),
    ("padded keys kept for local rows", "local[b, h, i] &= valid[b]", "pass"),
    ("global rows see padded keys", "glob[b, h, i] = valid[b]", "glob[b, h, i] = True"),
    ("scale 1/d", "scale = 1.0 / np.sqrt(d)", "scale = 1.0 / d"),
    ("global rows through the local projections",
     "o_glob = _masked_attention(qg, kg, vg, gm, scale)",
     "o_glob = _masked_attention(q, k, v, gm, scale)"),
    ("local rows take the global values", "o_local = _masked_attention(q, k, v, lm, scale)",
     "o_local = _masked_attention(q, k, vg, lm, scale)"),
    ("rows without keys not zeroed", "p = torch.where(mask, p, torch.zeros_like(p))", "pass"),
    ("output gradient ignored", "(o * g).sum().backward()", "o.sum().backward()"),
    ("gradients returned under swapped names",
     'names = ("q", "k", "v", "qg", "kg", "vg")\n    return',
     'names = ("q", "k", "v", "kg", "qg", "vg")\n    return'),
    ("one dilation for every head", "_is_tap(i, j, window, dil[h], causal)",
     "_is_tap(i, j, window, dil[0], causal)"),
    ("batch 0's padding for every batch", "local[b, h, i] &= valid[b]",
     "local[b, h, i] &= valid[0]"),
    ("batch 0's global tokens for every batch", "gpos = [j for j in range(n) if isg[b, j]]",
     "gpos = [j for j in range(n) if isg[0, j]]"),
]


@pytest.mark.parametrize("label,old,new", BWD_MUTATIONS, ids=[m[0] for m in BWD_MUTATIONS])
def test_backward_pins_catch_mutation(label, old, new):
    assert _caught(tb, "bwd", _mutant(obw, old, new), BWD_PINS), \
        f"no pin caught the planted mistake: {label}"


ENC_PINS = [(getattr(te, n), ()) for n in dir(te) if n.startswith("test_")]

ENC_MUTATIONS = [
    ("GELU in its tanh approximation", "return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))",
     "return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))"),
    ("LayerNorm with the unbiased variance",
     "var = ((y - mean) ** 2).mean(axis=-1, keepdims=True)",
     "var = ((y - mean) ** 2).sum(axis=-1, keepdims=True) / (y.shape[-1] - 1)"),
    ("feed-forward residual dropped", "return layer_norm(y + h, gamma, beta, eps)",
     "return layer_norm(y, gamma, beta, eps)"),
    ("intermediate bias dropped", "a = a + np.asarray(b1, np.float64)", "a = a"),
    ("GELU skipped", "a = gelu(a)", "a = a"),
    ("attention residual dropped", 'w["w_o"], w["b_o"], x, w["ln1_gamma"]',
     'w["w_o"], w["b_o"], 0 * x, w["ln1_gamma"]'),
    ("the two LayerNorms' parameters swapped",
     'w["w_2"], w["b_2"], w["ln2_gamma"], w["ln2_beta"],',
     'w["w_2"], w["b_2"], w["ln1_gamma"], w["ln1_beta"],'),
    ("global queries through the local weights",
     'wqg = w["w_qg"] if w["w_qg"] is not None else np.zeros((hid, hid))',
     'wqg = w["w_qkv"][:hid]'),
    ("every layer takes the first layer's window", "window=windows[l],",
     "window=windows[0],"),
    ("attention ignores the padding", 'p["vg"], local_mask,\n                          global_mask,',
     'p["vg"], None,\n                          global_mask,'),
    ("every layer takes the first layer's dilations",
     "dil = None if dilations is None else dilations[l]",
     "dil = None if dilations is None else dilations[0]"),
]


@pytest.mark.parametrize("label,old,new", ENC_MUTATIONS, ids=[m[0] for m in ENC_MUTATIONS])
def test_encoder_pins_catch_mutation(label, old, new):
    assert _caught(te, "enc", _mutant(oenc, old, new), ENC_PINS), \
        f"no pin caught the planted mistake: {label}"


def test_unmutated_copies_pass_every_pin():
    # Control: a copy compiled the same way with nothing changed passes all
    # pins, so a caught mutant is caught because of its mistake.
    assert _caught(tb, "bwd", _mutant(obw, "import numpy as np", "import numpy as np"),
                   BWD_PINS) == []
    assert _caught(te, "enc", _mutant(oenc, "import numpy as np", "import numpy as np"),
                   ENC_PINS) == []


# ----------------------------------------------- projection / output oracle
import test_projection_oracle as tp  # noqa: E402
from oracle import projection as oproj  # noqa: E402

PROJ_PINS = [(getattr(tp, n), ()) for n in dir(tp) if n.startswith("test_")]

PROJ_MUTATIONS = [
    ("heads split in the wrong order", "return y.reshape(B, n, H, d).transpose(0, 2, 1, 3)",
     "return y.reshape(B, H, n, d)"),
    ("weight blocks used transposed", 'y = np.einsum("bni,oi->bno", x, wp)',
     'y = np.einsum("bni,io->bno", x, wp)'),
    ("every block takes the first block's bias",
     "[p * hid:(p + 1) * hid]\n        out[name]", "[0:hid]\n        out[name]"),
    ("projection blocks in reverse order", "wp = w[p * hid:(p + 1) * hid]",
     "wp = w[(4 - p) * hid:(5 - p) * hid]"),
    ("Qg through the stacked Q weights", "y = x[b, rows] @ wqg.T", "y = x[b, rows] @ w[:hid].T"),
    ("heads concatenated in the wrong order",
     "merged = a.transpose(0, 2, 1, 3).reshape(B, n, H * d)",
     "merged = a.reshape(B, n, H * d)"),
    ("output weights used transposed",
     'y = np.einsum("bni,oi->bno", merged, np.asarray(wo, dtype=np.float64))',
     'y = np.einsum("bni,io->bno", merged, np.asarray(wo, dtype=np.float64))'),
    ("residual dropped", "y = y + np.asarray(residual, dtype=np.float64)", "y = y"),
    ("eps outside the square root", "z = (y - mean) / np.sqrt(var + eps)",
     "z = (y - mean) / (np.sqrt(var) + eps)"),
    ("batch 0's global count for every batch", "g = int(counts[b])", "g = int(counts[0])"),
    ("batch 0's hidden states for every global row", "y = x[b, rows] @ wqg.T",
     "y = x[0, rows] @ wqg.T"),
    ("gamma and beta swapped",
     "return z * np.asarray(gamma, dtype=np.float64) + np.asarray(beta, dtype=np.float64)",
     "return z * np.asarray(beta, dtype=np.float64) + np.asarray(gamma, dtype=np.float64)"),
]


def _caught_proj(mutant):
    saved = (tp.projection_forward, tp.output_layer)
    tp.projection_forward, tp.output_layer = mutant.projection_forward, mutant.output_layer
    caught = []
    try:
        for fn, args in PROJ_PINS:
            try:
                fn(*args)
            except Exception as e:
                caught.append((fn.__name__, type(e).__name__))
    finally:
        tp.projection_forward, tp.output_layer = saved
    return caught


@pytest.mark.parametrize("label,old,new", PROJ_MUTATIONS, ids=[m[0] for m in PROJ_MUTATIONS])
def test_projection_pins_catch_mutation(label, old, new):
    assert _caught_proj(_mutant(oproj, old, new)), f"no pin caught the planted mistake: {label}"


def test_unmutated_projection_copy_passes_every_pin():
    assert _caught_proj(_mutant(oproj, "import numpy as np", "import numpy as np")) == []

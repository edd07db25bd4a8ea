"""Pins of the projection oracle (oracle/projection.py) to closed forms:
identity and scaled-identity weights, one-hot tokens, bias only, and the
global-row gather.  Each pin fails for a transposed weight, a wrong head
split, a wrong block order or a Qg row written at the wrong position."""
import numpy as np

from oracle.projection import PROJECTIONS, projection_forward

H, D = 3, 64
HID = H * D


def _gidx(B, n, lists):
    gidx = -np.ones((B, n), dtype=np.int32)
    counts = np.zeros(B, dtype=np.int32)
    for b, pos in enumerate(lists):
        gidx[b, :len(pos)] = sorted(pos)
        counts[b] = len(pos)
    return gidx, counts


def test_scaled_identity_blocks_give_the_input_split_into_heads():
    rng = np.random.default_rng(1)
    B, n = 2, 5
    x = rng.standard_normal((B, n, HID))
    scales = [1.0, 2.0, -1.0, 0.0, 0.5]
    w = np.concatenate([s * np.eye(HID) for s in scales])
    gidx, counts = _gidx(B, n, [[], []])
    out = projection_forward(x, w, None, np.eye(HID), None, gidx, counts, H=H)
    for s, name in zip(scales, PROJECTIONS):
        for b in range(B):
            for h in range(H):
                for i in range(n):
                    np.testing.assert_array_equal(out[name][b, h, i], s * x[b, i, h * D:(h + 1) * D])


def test_one_hot_token_picks_a_weight_column():
    rng = np.random.default_rng(2)
    B, n = 1, 4
    w = rng.standard_normal((5 * HID, HID))
    bias = rng.standard_normal(5 * HID)
    x = np.zeros((B, n, HID))
    x[0, 2, 7] = 1.0                          # token 2 is the unit vector e_7
    gidx, counts = _gidx(B, n, [[]])
    out = projection_forward(x, w, bias, np.eye(HID), None, gidx, counts, H=H)
    for p, name in enumerate(PROJECTIONS):
        col = w[p * HID:(p + 1) * HID, 7] + bias[p * HID:(p + 1) * HID]
        got = out[name][0, :, 2, :].reshape(HID)          # heads in order
        np.testing.assert_allclose(got, col, rtol=0, atol=1e-12)
        other = out[name][0, :, 1, :].reshape(HID)        # a zero token gives the bias
        np.testing.assert_allclose(other, bias[p * HID:(p + 1) * HID], rtol=0, atol=0)


def test_qg_only_at_global_rows_and_equal_to_q_with_the_same_weights():
    rng = np.random.default_rng(3)
    B, n = 2, 9
    x = rng.standard_normal((B, n, HID))
    w = rng.standard_normal((5 * HID, HID)) / np.sqrt(HID)
    bias = rng.standard_normal(5 * HID)
    gidx, counts = _gidx(B, n, [[0, 4, 8], [6]])
    sentinel = np.full((B, H, n, D), 7.0)
    out = projection_forward(x, w, bias, w[:HID], bias[:HID], gidx, counts, H=H,
                             qg_init=sentinel)
    for b, pos in enumerate([[0, 4, 8], [6]]):
        for i in range(n):
            if i in pos:
                np.testing.assert_allclose(out["qg"][b, :, i], out["q"][b, :, i], atol=1e-12)
            else:
                np.testing.assert_array_equal(out["qg"][b, :, i], sentinel[b, :, i])


def test_linearity_in_the_input():
    rng = np.random.default_rng(4)
    B, n = 1, 6
    w = rng.standard_normal((5 * HID, HID))
    x1, x2 = rng.standard_normal((2, B, n, HID))
    gidx, counts = _gidx(B, n, [[1]])
    o1 = projection_forward(x1, w, None, w[:HID], None, gidx, counts, H=H)
    o2 = projection_forward(x2, w, None, w[:HID], None, gidx, counts, H=H)
    o12 = projection_forward(2 * x1 - x2, w, None, w[:HID], None, gidx, counts, H=H)
    for name in PROJECTIONS + ("qg",):
        np.testing.assert_allclose(o12[name], 2 * o1[name] - o2[name], atol=1e-9)


# ------------------------------------------------------------ output layer
from oracle.projection import output_layer  # noqa: E402


def test_output_layer_alternating_row_normalises_to_plus_minus_one():
    B, n = 1, 2
    attn = np.zeros((B, H, n, D))
    row = np.array([1.0, -1.0] * (HID // 2))            # mean 0, population variance 1
    attn[0, :, 1, :] = row.reshape(H, D)
    z = output_layer(attn, np.eye(HID), None, np.zeros((B, n, HID)), np.ones(HID),
                     np.zeros(HID), eps=1e-5)
    np.testing.assert_allclose(z[0, 1], row / np.sqrt(1.0 + 1e-5), rtol=0, atol=1e-12)


def test_output_layer_concatenates_heads_in_order():
    # A ramp over the features of a token, spread across heads: with identity
    # weights the normalised row is the normalised ramp only if head h lands
    # at features [h*d, (h+1)*d).
    B, n = 1, 1
    ramp = np.arange(HID, dtype=np.float64)
    attn = ramp.reshape(1, H, 1, D)
    z = output_layer(attn, np.eye(HID), None, np.zeros((B, n, HID)), np.ones(HID),
                     np.zeros(HID), eps=0.0)
    want = (ramp - ramp.mean()) / ramp.std()
    np.testing.assert_allclose(z[0, 0], want, atol=1e-12)


def test_output_layer_bias_residual_and_affine():
    rng = np.random.default_rng(7)
    B, n = 2, 3
    attn = rng.standard_normal((B, H, n, D))
    wo = rng.standard_normal((HID, HID)) / np.sqrt(HID)
    bo = rng.standard_normal(HID)
    res = rng.standard_normal((B, n, HID))
    g, b = rng.standard_normal(HID), rng.standard_normal(HID)
    z = output_layer(attn, wo, bo, res, g, b)
    unit = output_layer(attn, wo, bo, res, np.ones(HID), np.zeros(HID))
    np.testing.assert_allclose(z, unit * g + b, atol=1e-12)
    # unit-scale rows: mean 0 and variance 1 / (1 + eps / var)
    np.testing.assert_allclose(unit.mean(axis=-1), 0.0, atol=1e-12)
    # adding a constant to every feature of the pre-norm sum changes nothing
    z2 = output_layer(attn, wo, bo + 5.0, res, g, b)
    np.testing.assert_allclose(z2, z, atol=1e-9)


def test_qg_takes_its_own_weights_one_hot():
    # A one-hot token at a global row picks column c of wqg (plus bqg); the
    # stacked Q block is a different matrix, so using it instead would show.
    rng = np.random.default_rng(8)
    B, n, c = 1, 4, 77
    x = np.zeros((B, n, HID))
    x[0, 2, c] = 1.0
    w = rng.standard_normal((5 * HID, HID))
    wqg = rng.standard_normal((HID, HID))
    bqg = rng.standard_normal(HID)
    gidx, counts = _gidx(B, n, [[2]])
    out = projection_forward(x, w, None, wqg, bqg, gidx, counts, H=H)
    np.testing.assert_array_equal(out["qg"][0, :, 2, :].reshape(HID), wqg[:, c] + bqg)


def test_output_layer_weight_orientation():
    # attention output one-hot in feature c: the pre-norm sum is column c of
    # wo. Column c alternates +-1 (normalises to +-1/sqrt(1+eps)); row c is a
    # ramp, so a transposed wo gives a different row.
    B, n, c = 1, 1, 5
    wo = np.tile(np.arange(HID, dtype=np.float64), (HID, 1))      # row r = ramp
    wo[:, c] = np.array([1.0, -1.0] * (HID // 2))                  # column c alternates
    attn = np.zeros((B, H, n, D))
    attn[0, c // D, 0, c % D] = 1.0
    z = output_layer(attn, wo, None, np.zeros((B, n, HID)), np.ones(HID), np.zeros(HID),
                     eps=1e-5)
    np.testing.assert_allclose(z[0, 0], wo[:, c] / np.sqrt(1.0 + 1e-5), rtol=0, atol=1e-12)


def test_output_layer_adds_the_residual():
    # Zero attention output and bias: the row is the normalised residual.
    B, n = 1, 2
    res = np.zeros((B, n, HID))
    res[0, 1] = np.array([1.0, -1.0] * (HID // 2))
    z = output_layer(np.zeros((B, H, n, D)), np.eye(HID), None, res, np.ones(HID),
                     np.zeros(HID), eps=1e-5)
    np.testing.assert_allclose(z[0, 1], res[0, 1] / np.sqrt(1.0 + 1e-5), rtol=0, atol=1e-12)

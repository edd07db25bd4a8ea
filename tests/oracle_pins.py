"""Pins that tie the fp64 oracle to something other than itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with an independent statement of the method:

  * torch's scaled_dot_product_attention in fp64 (a library routine) for the
    special cases that reduce to full, causal or explicitly masked attention;
  * the residue decomposition of a dilated window (a dilated head equals
    independent undilated windows over the subsequences x[r::dil]);
  * truncation of tail padding;
  * softmax rows summing to one;
  * hand-derived key sets and closed-form softmax values under tests/golden/;
  * numpy.flatnonzero for the global-index compaction.

The mutation test plants mistakes in a copy of the oracle and checks that at
least one of these pins fails for every planted mistake.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TOL = 1e-11


def _rand(shape, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def _six(B, H, n, d, seed):
    return [_rand((B, H, n, d), seed + t) for t in range(6)]


def _sdpa(q, k, v, mask=None, causal=False):
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, is_causal=causal)


def _close(a, b, what, tol=TOL):
    a = np.asarray(a)
    b = np.asarray(b)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert np.all(np.isfinite(a)), f"{what}: non-finite values"
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------- compaction
def pin_global_index(orc):
    rng = np.random.default_rng(7)
    for (B, n, dens) in [(1, 1, 1.0), (3, 17, 0.3), (2, 64, 0.0), (2, 100, 1.0), (4, 333, 0.05)]:
        gm = (rng.random((B, n)) < dens).astype(np.uint8)
        gm[gm > 0] = rng.integers(1, 256, size=int(gm.sum()), dtype=np.uint8)  # any nonzero
        gidx, counts = orc.global_index(gm)
        for b in range(B):
            ref = np.flatnonzero(gm[b])
            assert counts[b] == ref.size, "global count differs from flatnonzero"
            assert np.array_equal(gidx[b, :ref.size], ref), "global index differs from flatnonzero"
            assert np.all(gidx[b, ref.size:] == -1), "tail of the global index is not -1"


# ------------------------------------------------------- reductions to SDPA
def pin_full_attention(orc):
    """w >= 2n, dilation 1, no globals, no padding: plain full attention."""
    B, H, n, d = 2, 3, 37, 8
    q, k, v, qg, kg, vg = _six(B, H, n, d, 100)
    for w in (2 * n, 2 * n + 6):
        out = orc.forward(q, k, v, qg, kg, vg, window=w)
        _close(out, _sdpa(q, k, v).numpy(), f"full attention w={w}")


def pin_causal_full(orc):
    """Causal with w >= n: causal full attention."""
    B, H, n, d = 1, 2, 29, 16
    q, k, v, qg, kg, vg = _six(B, H, n, d, 200)
    for w in (n, n + 3):
        out = orc.forward(q, k, v, qg, kg, vg, window=w, causal=True)
        _close(out, _sdpa(q, k, v, causal=True).numpy(), f"causal full w={w}")


def _tap_mask(n, w, dil, causal):
    """Boolean [n, n] mask of window taps, placed tap by tap."""
    m = torch.zeros((n, n), dtype=torch.bool)
    for i in range(n):
        offs = range(0, -w, -1) if causal else range(-(w // 2), w // 2 + 1)
        for kk in offs:
            j = i + kk * dil
            if 0 <= j < n:
                m[i, j] = True
    return m


def pin_band_masked(orc):
    """No globals: equals attention with an explicit mask of window taps."""
    B, H, n, d = 1, 2, 41, 8
    q, k, v, qg, kg, vg = _six(B, H, n, d, 300)
    for (w, dil, causal) in [(6, 1, False), (10, 1, False), (2, 1, False), (6, 3, False),
                             (4, 2, False), (5, 1, True), (7, 2, True), (1, 1, True)]:
        out = orc.forward(q, k, v, qg, kg, vg, window=w, dilation=[dil] * H, causal=causal)
        ref = _sdpa(q, k, v, mask=_tap_mask(n, w, dil, causal)).numpy()
        _close(out, ref, f"band w={w} dil={dil} causal={causal}")


def pin_globals_masked(orc):
    """Globals at arbitrary positions: local rows equal attention over
    (taps OR global column) with K, V; global rows equal full attention with
    Qg, Kg, Vg."""
    B, H, n, d = 2, 2, 45, 8
    q, k, v, qg, kg, vg = _six(B, H, n, d, 400)
    gpos = [[0, 7, 8, 30, 44], [3, 21]]
    gm = torch.zeros((B, n), dtype=torch.uint8)
    for b, ps in enumerate(gpos):
        gm[b, ps] = 1
    for (w, dil) in [(4, 1), (8, 2), (2, 3), (2 * n, 1)]:
        out = orc.forward(q, k, v, qg, kg, vg, None, gm, window=w, dilation=[dil] * H)
        for b in range(B):
            m = _tap_mask(n, w, dil, False)
            m[:, gpos[b]] = True
            loc = _sdpa(q[b], k[b], v[b], mask=m).numpy()
            glo = _sdpa(qg[b], kg[b], vg[b]).numpy()
            for i in range(n):
                ref = glo[:, i] if i in gpos[b] else loc[:, i]
                _close(out[b, :, i], ref, f"globals w={w} dil={dil} b={b} row {i}")


def pin_full_with_globals(orc):
    """w >= 2n with globals: a global key already in the window must not be
    counted twice, so local rows equal plain full attention."""
    B, H, n, d = 1, 2, 33, 8
    q, k, v, qg, kg, vg = _six(B, H, n, d, 500)
    gm = torch.zeros((B, n), dtype=torch.uint8)
    gm[0, [1, 16, 32]] = 1
    out = orc.forward(q, k, v, qg, kg, vg, None, gm, window=2 * n)
    loc = _sdpa(q, k, v).numpy()
    glo = _sdpa(qg, kg, vg).numpy()
    for i in range(n):
        ref = glo[0, :, i] if gm[0, i] else loc[0, :, i]
        _close(out[0, :, i], ref, f"full+globals row {i}")


def pin_per_head_dilation(orc):
    """Each head takes its own dilation (LF-notes, Dilated Sliding Window:
    different dilations per head): every (batch, head) equals attention with
    an explicit tap mask of that head's dilation."""
    B, H, n, d = 2, 3, 37, 8
    q, k, v, qg, kg, vg = _six(B, H, n, d, 350)
    dils = [1, 3, 2]
    for (w, causal) in [(6, False), (5, True)]:
        out = orc.forward(q, k, v, qg, kg, vg, window=w, dilation=dils, causal=causal)
        for b in range(B):
            for h in range(H):
                ref = _sdpa(q[b, h], k[b, h], v[b, h],
                            mask=_tap_mask(n, w, dils[h], causal)).numpy()
                _close(out[b, h], ref, f"per-head dilation w={w} b={b} h={h} causal={causal}")


# ------------------------------------------------------ structural identities
def pin_dilation_residue(orc):
    """A head with dilation dil equals dil independent undilated windows over
    the residue subsequences x[r::dil]."""
    B, H, n, d = 1, 1, 53, 8
    q, k, v, qg, kg, vg = _six(B, H, n, d, 600)
    for (w, dil, causal) in [(4, 2, False), (6, 3, False), (3, 2, True), (5, 4, True)]:
        out = orc.forward(q, k, v, qg, kg, vg, window=w, dilation=[dil], causal=causal)
        for r in range(dil):
            sub = [t[:, :, r::dil].contiguous() for t in (q, k, v, qg, kg, vg)]
            ref = orc.forward(*sub, window=w, dilation=[1], causal=causal)
            _close(out[:, :, r::dil], ref, f"residue w={w} dil={dil} r={r} causal={causal}")


def pin_padding_truncation(orc):
    """Tail padding: valid rows equal the run on the truncated sequence, padded
    rows are exactly zero (also when a padded position is marked global)."""
    B, H, n, d, pad = 1, 2, 40, 8, 11
    q, k, v, qg, kg, vg = _six(B, H, n, d, 700)
    lm = torch.ones((B, n), dtype=torch.uint8)
    lm[0, n - pad:] = 0
    gm = torch.zeros((B, n), dtype=torch.uint8)
    gm[0, [2, 20, n - 3]] = 1          # n-3 is padded and global
    for (w, dil) in [(6, 1), (4, 2), (2 * n, 1)]:
        out = orc.forward(q, k, v, qg, kg, vg, lm, gm, window=w, dilation=[dil] * H)
        t = n - pad
        sub = [x[:, :, :t].contiguous() for x in (q, k, v, qg, kg, vg)]
        ref = orc.forward(*sub, None, gm[:, :t].contiguous(), window=w, dilation=[dil] * H)
        _close(out[:, :, :t], ref, f"padding w={w} dil={dil}")
        assert np.all(out[:, :, t:] == 0.0), "padded rows are not zero"
    for causal_w in (5, 64):
        out = orc.forward(q, k, v, qg, kg, vg, lm, None, window=causal_w, causal=True)
        sub = [x[:, :, :n - pad].contiguous() for x in (q, k, v, qg, kg, vg)]
        ref = orc.forward(*sub, window=causal_w, causal=True)
        _close(out[:, :, :n - pad], ref, f"causal padding w={causal_w}")
        assert np.all(out[:, :, n - pad:] == 0.0), "padded causal rows are not zero"


def pin_row_sums(orc):
    """Every probability row sums to one over unique, valid keys."""
    B, H, n, d = 2, 2, 50, 8
    q, k, v, qg, kg, vg = _six(B, H, n, d, 800)
    lm = torch.ones((B, n), dtype=torch.uint8)
    lm[1, 38:] = 0
    gm = torch.zeros((B, n), dtype=torch.uint8)
    gm[:, [0, 25]] = 1
    for (w, dil) in [(8, 1), (6, 3)]:
        for b in range(B):
            for h in range(H):
                for i in range(n):
                    keys, probs = orc.row_probs(q, k, qg, kg, lm, gm, window=w,
                                                dilation=[dil] * H, b=b, h=h, i=i)
                    if lm[b, i] == 0:
                        assert keys.size == 0, "a padded row has keys"
                        continue
                    assert keys.size == np.unique(keys).size, "a key is counted twice"
                    assert np.all(lm[b, keys.astype(np.int64)].numpy() == 1), "padded key used"
                    assert np.all(probs > 0), "non-positive probability"
                    assert abs(probs.sum() - 1.0) <= 1e-12, "row does not sum to one"


# ------------------------------------------------------------------ golden
def load_key_set_cases():
    cases = []
    cur = None
    with open(os.path.join(GOLDEN, "key_sets.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if line.startswith("case "):
                parts = line.split()
                kv = dict(p.split("=", 1) for p in parts[2:])
                cur = dict(name=parts[1], n=int(kv["n"]), w=int(kv["w"]), dil=int(kv["dil"]),
                           causal=kv["causal"] == "1",
                           globals=[] if kv["globals"] == "-" else
                           [int(x) for x in kv["globals"].split(",")],
                           pad_tail=int(kv["pad_tail"]), rows={})
                cases.append(cur)
            elif line.startswith("row "):
                head, _, rest = line.partition(":")
                i = int(head.split()[1])
                rest = rest.strip()
                cur["rows"][i] = set() if rest == "-" else {int(x) for x in rest.split()}
    return cases


def _case_masks(c):
    n = c["n"]
    lm = torch.ones((1, n), dtype=torch.uint8)
    if c["pad_tail"]:
        lm[0, n - c["pad_tail"]:] = 0
    gm = None
    if c["globals"]:
        gm = torch.zeros((1, n), dtype=torch.uint8)
        gm[0, c["globals"]] = 1
    return lm, gm


def pin_golden_key_sets(orc):
    for c in load_key_set_cases():
        n = c["n"]
        q, k, v, qg, kg, vg = _six(1, 1, n, 4, 900)
        lm, gm = _case_masks(c)
        for i, want in c["rows"].items():
            keys, _ = orc.row_probs(q, k, qg, kg, lm, gm, window=c["w"], dilation=[c["dil"]],
                                    causal=c["causal"], i=i)
            assert set(int(x) for x in keys) == want, \
                f"key set of {c['name']} row {i}: {sorted(keys)} != {sorted(want)}"


def pin_uniform_closed_form(orc):
    """Q = Qg = 0 makes every score equal, so each row is the plain mean of
    the value rows of its key set; with V = Vg = identity the output row is
    the indicator of the key set divided by its size."""
    for c in load_key_set_cases():
        n = c["n"]
        z = torch.zeros((1, 1, n, n), dtype=torch.float64)
        eye = torch.eye(n, dtype=torch.float64).reshape(1, 1, n, n)
        kk = _rand((1, 1, n, n), 901)
        lm, gm = _case_masks(c)
        out = orc.forward(z, kk, eye, z, kk, eye, lm, gm, window=c["w"], dilation=[c["dil"]],
                          causal=c["causal"])
        for i, want in c["rows"].items():
            ref = np.zeros(n)
            if want:
                ref[sorted(want)] = 1.0 / len(want)
            _close(out[0, 0, i], ref, f"uniform {c['name']} row {i}", tol=1e-14)


def pin_closed_form_examples(orc):
    env = {"log": math.log, "__builtins__": {}}
    with open(os.path.join(GOLDEN, "closed_form.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        n, d = c["n"], c["d"]

        def dense(key):
            t = torch.zeros((1, 1, n, d), dtype=torch.float64)
            for row, vals in c.get(key, {}).items():
                t[0, 0, int(row)] = torch.tensor([eval(x, env) for x in vals], dtype=torch.float64)
            return t

        gm = None
        if c["globals"]:
            gm = torch.zeros((1, n), dtype=torch.uint8)
            gm[0, c["globals"]] = 1
        out = orc.forward(dense("q"), dense("k"), dense("v"), dense("qg"), dense("kg"),
                          dense("vg"), None, gm, window=c["window"],
                          dilation=[c["dilation"]], causal=c["causal"])
        for row, vals in c["expect"].items():
            ref = np.array([eval(x, env) for x in vals])
            _close(out[0, 0, int(row)], ref, f"closed form '{c['name']}' row {row}", tol=1e-12)


def pin_rejects_causal_globals(orc):
    q, k, v, qg, kg, vg = _six(1, 1, 8, 4, 950)
    gm = torch.zeros((1, 8), dtype=torch.uint8)
    gm[0, 3] = 1
    try:
        orc.forward(q, k, v, qg, kg, vg, None, gm, window=4, causal=True)
    except RuntimeError:
        return
    raise AssertionError("causal attention with global tokens was accepted")


ALL_PINS = [pin_global_index, pin_full_attention, pin_causal_full, pin_band_masked,
            pin_per_head_dilation, pin_globals_masked, pin_full_with_globals, pin_dilation_residue,
            pin_padding_truncation, pin_row_sums, pin_golden_key_sets,
            pin_uniform_closed_form, pin_closed_form_examples, pin_rejects_causal_globals]

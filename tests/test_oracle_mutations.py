"""Plant plausible mistakes in a private copy of the oracle and check that the
pins catch every one of them (CPU only; the committed oracle is untouched)."""
import os

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "lf_oracle.c")

# (label, exact text in lf_oracle.c, replacement)
MUTATIONS = [
    ("window one tap short on the right", "k <= w / 2; ++k)", "k < w / 2; ++k)"),
    ("window one tap short on the left", "int k = -(w / 2);", "int k = -(w / 2) + 1;"),
    ("dilation ignored", "long j = (long)i + (long)k * dil;", "long j = (long)i + (long)k;"),
    ("causal looks right", "long j = (long)i - (long)k * dil;", "long j = (long)i + (long)k * dil;"),
    ("causal window one tap long", "for (int k = w - 1; k >= 0; --k)", "for (int k = w; k >= 0; --k)"),
    ("global key counted twice", "if (in_window(i, j, w, dil, causal)) continue;", ""),
    ("dedupe ignores dilation", "if (a % dil != 0) return 0;", ""),
    ("global columns dropped", "for (int t = 0; t < g; ++t) {", "for (int t = 0; t < 0; ++t) {"),
    ("global rows use K", "softmax_attend(qg + base + (size_t)i * d, kg + base, vg + base",
     "softmax_attend(qg + base + (size_t)i * d, k + base, vg + base"),
    ("global rows use Q", "softmax_attend(qg + base + (size_t)i * d, kg + base, vg + base",
     "softmax_attend(q + base + (size_t)i * d, kg + base, vg + base"),
    ("local rows use Vg", "softmax_attend(q + base + (size_t)i * d, k + base, v + base",
     "softmax_attend(q + base + (size_t)i * d, k + base, vg + base"),
    ("global rows treated as local", "if (gm_b && gm_b[i] != 0) {                    /* global row */",
     "if (0) {"),
    ("padded rows not zeroed", "if (!is_valid_key(lm_b, i)) {                 /* R6: padded row */",
     "if (0) {"),
    ("padded keys used", "return local_mask_b == NULL || local_mask_b[j] != 0;", "return 1;"),
    ("scale 1/d", "const double scale = 1.0 / sqrt((double)d);", "const double scale = 1.0 / (double)d;"),
    ("value row index transposed", "const double *vrow = vmat + (size_t)keys[t] * d;",
     "const double *vrow = vmat + (size_t)t * d;"),
    ("denominator squared", "denom += scores[t];", "denom += scores[t] * scores[t];"),
    ("global index shifted", "global_idx[(size_t)b * n + cnt] = p;",
     "global_idx[(size_t)b * n + cnt] = (p > 0 ? p - 1 : p);"),
    ("last global dropped", "counts[b] = cnt;", "counts[b] = cnt > 0 ? cnt - 1 : 0;"),
    ("dot product drops a term", "for (int x = 0; x < d; ++x) dot += qrow[x] * krow[x];",
     "for (int x = 1; x < d; ++x) dot += qrow[x] * krow[x];"),
    ("padded global keys used by local rows",
     "        if (!is_valid_key(local_mask_b, j)) continue;\n        if (in_window",
     "        if (in_window"),
    ("dedupe window too wide", "return a / dil <= w / 2;", "return a / dil <= w;"),
    ("batch 0's global index for every batch", "gidx + (size_t)b * n, cnts[b]", "gidx, cnts[0]"),
    ("batch 0's global mask for every batch",
     "const uint8_t *gm_b = global_mask ? global_mask + (size_t)b * n : NULL;",
     "const uint8_t *gm_b = global_mask ? global_mask : NULL;"),
    ("batch 0's local mask for every batch",
     "const uint8_t *lm_b = local_mask ? local_mask + (size_t)b * n : NULL;",
     "const uint8_t *lm_b = local_mask ? local_mask : NULL;"),
    ("dilation indexed by batch", "int dil = dilation ? dilation[h] : 1;",
     "int dil = dilation ? dilation[b] : 1;"),
    ("one dilation for every head", "int dil = dilation ? dilation[h] : 1;",
     "int dil = dilation ? dilation[0] : 1;"),
    ("tensor base ignores the batch", "size_t base = (size_t)bh * n * d;",
     "size_t base = (size_t)h * n * d;"),
]


@pytest.mark.parametrize("label,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(tmp_path, label, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation target not found: {old!r}"
    mutated = tmp_path / "lf_oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    lib_path = oracle.build(str(mutated), str(tmp_path / "liblf_oracle_mut.so"), force=True)
    orc = oracle.Oracle(oracle.load(lib_path))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, RuntimeError) as e:
            caught.append((pin.__name__, str(e)[:80]))
    assert caught, f"no pin caught the planted mistake: {label}"

"""Work accounting against the oracle's own key sets (CPU only)."""
import numpy as np
import pytest

import oracle
from sparse_long_sequence_lf_b200 import accounting
from sparse_long_sequence_lf_b200.workloads import WORKLOADS, Workload, make_inputs, \
    random_workload


def _pairs_by_oracle(wl):
    x = make_inputs(wl)
    total = 0
    for b in range(wl.B):
        for h in range(wl.H):
            for i in range(wl.n):
                keys, _ = oracle.row_probs(x["q"], x["k"], x["qg"], x["kg"], x["local_mask"],
                                           x["global_mask"], window=wl.window,
                                           dilation=x["dilation"], causal=wl.causal,
                                           b=b, h=h, i=i)
                total += keys.size
    return total


CASES = [
    Workload("a", "bf16", 1, 2, 37, 8, dilation=(1, 3), globals_kind="list:0,20"),
    Workload("b", "f16", 2, 1, 50, 6, globals_kind="list:3,49;10", pad_tail=(0, 12)),
    Workload("c", "bf16", 1, 3, 45, 5, dilation=(1, 2, 4), causal=True, pad_tail=(7,)),
    Workload("d", "f32", 1, 1, 30, 100, globals_kind="first:4"),
]


@pytest.mark.parametrize("wl", CASES, ids=[c.name for c in CASES])
def test_pairs_equal_oracle_key_sets(wl):
    assert accounting.useful_pairs(wl) == _pairs_by_oracle(wl)


def test_random_pairs_equal_oracle_key_sets():
    rng = np.random.default_rng(5)
    for t in range(4):
        wl = random_workload(rng, max_n=60, name=f"r{t}")
        assert accounting.useful_pairs(wl) == _pairs_by_oracle(wl)


def test_headline_workload_figures():
    wl = WORKLOADS["bf16-b1h12-n4096-w512-g1"]
    flops = accounting.useful_flops(wl)
    assert 6.2e9 < flops < 6.4e9
    assert accounting.algorithmic_bytes(wl) == 6 * 12 * 4096 * 64 * 2 + 12 * 64 * 2


def test_backward_flops_are_ten_d_per_pair():
    wl = CASES[0]
    assert accounting.backward_flops(wl) == 10 * wl.d * accounting.useful_pairs(wl)
    assert accounting.backward_flops(wl) == 2.5 * accounting.useful_flops(wl)


def test_encoder_flops_count_every_product_of_a_layer():
    import bench
    from sparse_long_sequence_lf_b200.workloads import EncoderWorkload
    wl = Workload("e", "f16", 1, 2, 40, 8, globals_kind="list:0,17")
    ew = EncoderWorkload("enc", wl, inter=256, layers=3)
    hid, tok, g = 128, 40, 2
    per_layer = (2 * tok * hid * 5 * hid          # Q, K, V, Kg, Vg
                 + 2 * g * hid * hid              # Qg of the global rows
                 + accounting.useful_flops(wl)    # the attention
                 + 2 * tok * hid * hid            # output projection
                 + 2 * tok * hid * 256            # FFN intermediate
                 + 2 * tok * 256 * hid)           # FFN output
    assert bench.encoder_flops(ew, [g]) == 3 * per_layer


@pytest.mark.parametrize("wl", CASES, ids=[c.name for c in CASES])
def test_row_block_flops_add_up(wl):
    # Row blocks of every (batch, head) partition the whole count.
    total = 0
    for b in range(wl.B):
        for h in range(wl.H):
            cut = wl.n // 3
            total += accounting.useful_flops_rows(wl, h, (0, cut), batch=b)
            total += accounting.useful_flops_rows(wl, h, (cut, wl.n), batch=b)
    assert total == accounting.useful_flops(wl)

"""Parity of the feed-forward block and of the encoder stack (CUDA, through
the C ABI) with the fp64 oracle of oracle/encoder.py.

Tolerance: |got - want| <= 2e-2 * max(1, |want|) per element for bf16 and
fp16.  The layer outputs are LayerNorm outputs of magnitude up to about 4,
where one bf16 rounding alone is up to 2^-7; the relative part covers that,
the absolute part the fp32 sums of products of rounded operands.
"""
import numpy as np
import pytest
import torch

import sparse_long_sequence_lf_b200 as lf
from oracle import encoder as oenc
from sparse_long_sequence_lf_b200.workloads import Workload, make_encoder_inputs, make_masks

pytestmark = pytest.mark.gpu

TOL = 2e-2


def check(got, want, what):
    got = got.float().cpu().numpy().astype(np.float64)
    assert got.shape == want.shape, what
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    excess = np.abs(got - want) - TOL * np.maximum(1.0, np.abs(want))
    worst = np.unravel_index(int(np.argmax(excess)), excess.shape)
    assert excess.max() <= 0, (f"{what}: err {abs(got[worst] - want[worst]):.3e} at {worst}: "
                               f"got {got[worst]:.5f} want {want[worst]:.5f}")


FFN_CASES = [
    ("bf16", 1, 300, 128, 512),
    ("f16", 2, 200, 768, 3072),
    ("bf16", 1, 129, 1280, 256),      # > 1024 features: the multi-pass LayerNorm
    ("bf16", 3, 64, 64, 64),
]


@pytest.mark.parametrize("dt,B,n,hidden,inter", FFN_CASES)
def test_ffn_block(dt, B, n, hidden, inter):
    wl = Workload("ffn", dt, B, hidden // 64, n, 2, seed=B * 1000 + n)
    x, layers = make_encoder_inputs(wl, 1, inter)
    lw = layers[0]
    dev = {k: v.cuda() for k, v in lw.items()}
    out = lf.ffn_block(x.cuda(), dev["w_1"], dev["b_1"], dev["w_2"], dev["b_2"],
                       dev["ln2_gamma"], dev["ln2_beta"])
    torch.cuda.synchronize()
    want = oenc.ffn_block(x.double().numpy(), *(lw[k].double().numpy() for k in
                                               ("w_1", "b_1", "w_2", "b_2", "ln2_gamma",
                                                "ln2_beta")))
    check(out, want, f"ffn {dt} B{B} n{n} {hidden}x{inter}")


def test_ffn_without_biases():
    wl = Workload("ffn-nob", "bf16", 1, 2, 150, 2, seed=3)
    x, layers = make_encoder_inputs(wl, 1, 256)
    lw = {k: v.cuda() for k, v in layers[0].items()}
    out = lf.ffn_block(x.cuda(), lw["w_1"], None, lw["w_2"], None, lw["ln2_gamma"],
                       lw["ln2_beta"])
    torch.cuda.synchronize()
    c = {k: v.double().numpy() for k, v in layers[0].items()}
    want = oenc.ffn_block(x.double().numpy(), c["w_1"], None, c["w_2"], None, c["ln2_gamma"],
                          c["ln2_beta"])
    check(out, want, "ffn without biases")


ENC_CASES = [
    # (workload, layers, inter, windows, dilations)
    (Workload("enc-g-pad", "bf16", 2, 2, 500, 64, globals_kind="list:3,480;7,499",
              pad_tail=(30, 1), seed=21), 1, 512, [64], None),
    (Workload("enc-nog", "bf16", 1, 4, 384, 32, seed=22), 1, 1024, [32], [[1, 2, 1, 3]]),
    (Workload("enc-3layers", "f16", 1, 2, 700, 16, globals_kind="random:5", seed=23), 3, 256,
     [16, 64, 128], [[1, 1], [2, 1], [1, 3]]),
    # one layer of the benchmark model at full width (16 heads, hidden 1024,
    # intermediate 4096, window 512, 64 global tokens at the front), 1024 tokens
    (Workload("enc-full-width", "f16", 1, 16, 1024, 512, globals_kind="first:64", seed=25), 1,
     4096, [512], None),
]


@pytest.mark.parametrize("case", ENC_CASES, ids=[c[0].name for c in ENC_CASES])
def test_encoder_stack(case):
    wl, L, inter, windows, dils = case
    x, layers = make_encoder_inputs(wl, L, inter)
    local, glob = make_masks(wl)
    dev_layers = [{k: v.cuda() for k, v in lw.items()} for lw in layers]
    out = lf.encoder_forward(x.cuda(), dev_layers, None if local is None else local.cuda(),
                             None if glob is None else glob.cuda(), H=wl.H, windows=windows,
                             dilations=dils)
    torch.cuda.synchronize()
    rnd = lambda a: torch.from_numpy(a).to(wl.torch_dtype).double().numpy()
    want = oenc.encoder_forward(x, [{k: v.double().numpy() for k, v in lw.items()}
                                    for lw in layers], local, glob, H=wl.H, windows=windows,
                                dilations=dils, round_to=rnd)
    check(out, want, wl.name)


def test_encoder_status_and_arg_checks():
    wl = Workload("enc-args", "bf16", 1, 2, 256, 32, seed=24)
    x, layers = make_encoder_inputs(wl, 2, 256)
    dev_layers = [{k: v.cuda() for k, v in lw.items()} for lw in layers]
    ws = torch.empty(lf.encoder_workspace_size(1, 256, 2, 256, 0), dtype=torch.uint8,
                     device="cuda")
    lf.encoder_forward(x.cuda(), dev_layers, H=2, windows=[32, 64], max_global=0, workspace=ws)
    assert lf.workspace_status(ws) == 0
    with pytest.raises(lf.LfError):          # odd window in the second layer
        lf.encoder_forward(x.cuda(), dev_layers, H=2, windows=[32, 63], max_global=0,
                           workspace=ws)
    with pytest.raises(lf.LfError):          # workspace too small
        lf.encoder_forward(x.cuda(), dev_layers, H=2, windows=[32, 64], max_global=0,
                           workspace=ws[:1024])

"""The no-allocation entry point, lf_attention_forward_static, called through
the C ABI and compared with lf_attention_forward on the same inputs.

This file is collected last on purpose: the static scratch is one array per
device, and the first call on a device does its one-time set-up, so these
tests must pass both in a fresh process and after every other test.
"""
import pytest
import torch

import sparse_long_sequence_lf_b200 as lf
from sparse_long_sequence_lf_b200._lib import STATIC_SCRATCH_BYTES
from sparse_long_sequence_lf_b200.workloads import Workload, make_inputs
from gpu_helpers import TOL, assert_close, max_global_of, oracle_forward, to_dev

CASES = [
    # globals anywhere, tail padding, per-head dilation
    Workload("static-bf16-b2h3-n700", "bf16", 2, 3, 700, 64, dilation=(1, 2, 3),
             globals_kind="list:0,5,350,699;13,200", pad_tail=(0, 123), seed=71),
    Workload("static-f16-b1h4-n1500", "f16", 1, 4, 1500, 256, globals_kind="random:9",
             seed=72),
    Workload("static-f32-b1h2-n513", "f32", 1, 2, 513, 64, globals_kind="first:2",
             pad_tail=(7,), seed=73),
]


@pytest.mark.gpu
@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_static_scratch_matches_forward(wl):
    x = make_inputs(wl)
    g = to_dev(x)
    mg = max_global_of(x)
    args = (g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"], g["local_mask"],
            g["global_mask"])
    kw = dict(window=x["window"], dilation=x["dilation"], causal=x["causal"], max_global=mg)
    ref = lf.attention_forward(*args, **kw)
    outs = [torch.full_like(g["q"], float("nan")) for _ in range(2)]
    scratch = []
    for out in outs:                       # two calls in a row
        scratch.append(lf.attention_forward_static(*args, out=out, **kw))
    torch.cuda.synchronize()
    assert scratch[0] == scratch[1] != 0
    assert lf.scratch_status(scratch[1]) == 0
    # The same kernels on the same inputs: the results must be identical, bit
    # for bit; a scratch region that aliased another would show here.
    for out in outs:
        assert torch.equal(out, ref)
    # And the static path on its own against the fp64 oracle.
    assert_close(outs[1], oracle_forward(x), TOL[wl.dtype], wl.name)


def test_static_scratch_limit_is_refused():
    # B=1, H=64, n=65536 with 64 global tokens needs ~142 MB of workspace: the
    # C entry refuses it before anything touches a device (no GPU needed).
    from sparse_long_sequence_lf_b200 import _lib
    need = lf.workspace_size(1, 64, 65536, 64)
    assert need > STATIC_SCRATCH_BYTES
    rc = _lib.lib().lf_attention_forward_static(
        _lib.LF_BF16, 1, 64, 65536, 64, None, None, None, None, None, None, None, None, 64,
        512, None, 0, None, None, None)
    assert rc == -8
    assert b"16 MiB" in _lib.lib().lf_status_string(rc)


@pytest.mark.parametrize("sizes,code", [((0, 2, 256, 64, 1), -1), ((1, 2, 256, 64, 300), -1),
                                        ((1, 2, 256, 32, 1), -2)])
def test_static_invalid_sizes_are_refused_on_the_host(sizes, code):
    # Sizes with no workspace are refused before anything touches a device
    # (no GPU needed): zero batches, more global slots than tokens, d_head 32.
    from sparse_long_sequence_lf_b200 import _lib
    B, H, n, d, mg = sizes
    rc = _lib.lib().lf_attention_forward_static(
        _lib.LF_BF16, B, H, n, d, None, None, None, None, None, None, None, None, mg,
        64, None, 0, None, None, None)
    assert rc == code

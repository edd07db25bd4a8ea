"""Host-side argument checks of the Python binding that need no GPU: wrong
shapes, dtypes or devices are refused before anything reaches the library."""
import pytest
import torch

import sparse_long_sequence_lf_b200 as lf


def test_attention_forward_rejects_bad_projections():
    q = torch.zeros(1, 2, 16, 64)
    with pytest.raises((TypeError, ValueError)):
        lf.attention_forward(q.to(torch.int32), q, q, q, q, q, window=4, max_global=0)
    with pytest.raises(ValueError):
        lf.attention_forward(q[..., :32], q, q, q, q, q, window=4, max_global=0)
    with pytest.raises(ValueError):                       # CPU tensors
        lf.attention_forward(q, q, q, q, q, q, window=4, max_global=0)


def test_attention_backward_rejects_mismatched_tensors():
    q = torch.zeros(1, 2, 16, 64)
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError):
        lf.attention_backward(q, q, q, q, q, q, q[:, :1], q, window=4, max_global=0,
                              workspace=ws)
    with pytest.raises(ValueError):                       # CPU tensors
        lf.attention_backward(q, q, q, q, q, q, q, q, window=4, max_global=0, workspace=ws)


def test_ffn_block_rejects_bad_inputs():
    h = torch.zeros(1, 8, 64, dtype=torch.bfloat16)
    w1 = torch.zeros(128, 64, dtype=torch.bfloat16)
    w2 = torch.zeros(64, 128, dtype=torch.bfloat16)
    g = torch.zeros(64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):                       # fp32 input
        lf.ffn_block(h.float(), w1, None, w2, None, g, g)
    with pytest.raises(ValueError):                       # CPU tensors
        lf.ffn_block(h, w1, None, w2, None, g, g)


def test_encoder_forward_rejects_bad_inputs():
    x = torch.zeros(1, 8, 128, dtype=torch.float16)
    layer = {"w_1": torch.zeros(256, 128, dtype=torch.float16)}
    with pytest.raises(ValueError):                       # last dim must be H*64
        lf.encoder_forward(x, [layer], H=3, windows=[4])
    with pytest.raises(ValueError):                       # one window per layer
        lf.encoder_forward(x, [layer, layer], H=2, windows=[4])
    with pytest.raises(ValueError):                       # fp32 input
        lf.encoder_forward(x.float(), [layer], H=2, windows=[4])
    with pytest.raises(ValueError):                       # CPU weights
        lf.encoder_forward(x, [layer], H=2, windows=[4])


def test_buffers_must_be_device_tensors():
    # A host buffer would reach the kernels as a device address: refused first.
    from sparse_long_sequence_lf_b200.api import _dev
    assert _dev(None, "x") is None
    with pytest.raises(ValueError):
        _dev(torch.zeros(4), "workspace")
    with pytest.raises(ValueError):
        _dev([1, 2], "workspace")
    with pytest.raises(ValueError):
        lf.workspace_status(torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(ValueError):
        lf.attention_prepare(None, None, B=1, H=1, n=8, max_global=0,
                             workspace=torch.zeros(1024, dtype=torch.uint8))

"""Python binding of the C ABI in include/lf_attention.h.

Argument marshalling only: shapes and dtypes are checked, pointers and the
current CUDA stream are handed to the library, and every step of the
attention runs in the library's CUDA kernels.  PyTorch provides device memory
and streams.  There is no CPU fallback: without the built library (or
without an sm_100 GPU) every call raises.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import LF_BF16, LF_F16, LF_F32, LfError

D_HEAD = 64
_DTYPES = {torch.float32: LF_F32, torch.float16: LF_F16, torch.bfloat16: LF_BF16}


def _stream_ptr(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _mask(m, B, n, name):
    if m is None:
        return None
    if m.dtype == torch.bool:
        m = m.view(torch.uint8)
    if m.dtype != torch.uint8:
        raise TypeError(f"{name} must be uint8 or bool")
    if tuple(m.shape) != (B, n) or not m.is_contiguous() or not m.is_cuda:
        raise ValueError(f"{name} must be a contiguous CUDA tensor of shape [B, n]")
    return m


def _dilation(dilation, H):
    if dilation is None:
        return None
    vals = [int(x) for x in (dilation.tolist() if hasattr(dilation, "tolist") else dilation)]
    if len(vals) != H:
        raise ValueError("dilation must have one entry per head")
    return (ctypes.c_int32 * H)(*vals)


def _dev(t, name, dtype=None, shape=None):
    """A buffer handed to the library: a contiguous CUDA tensor (host memory
    would reach the kernels as a device address); None passes through."""
    if t is None:
        return None
    if not torch.is_tensor(t) or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}")
    return t


def _check_projections(tensors):
    q = tensors[0]
    if q.dtype not in _DTYPES:
        raise TypeError("projections must be float32, float16 or bfloat16")
    if q.dim() != 4 or q.shape[-1] != D_HEAD:
        raise ValueError("projections must have shape [B, H, n, 64]")
    for t in tensors:
        if t.dtype != q.dtype or t.shape != q.shape:
            raise ValueError("all projections must share dtype and shape")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("projections must be contiguous CUDA tensors")
    return _DTYPES[q.dtype], q.shape


def workspace_size(B: int, H: int, n: int, max_global: int) -> int:
    size = _lib.lib().lf_workspace_size(B, H, n, D_HEAD, max_global)
    if size == 0:
        raise LfError(-1, "lf_workspace_size")
    return int(size)


def new_workspace(B: int, H: int, n: int, max_global: int, device=None) -> torch.Tensor:
    return torch.empty(workspace_size(B, H, n, max_global), dtype=torch.uint8,
                       device=device or "cuda")


def global_index(global_mask: torch.Tensor, stream=None):
    """Compacted global positions per batch (ascending, -1 padded) and counts."""
    B, n = global_mask.shape
    gm = _mask(global_mask, B, n, "global_mask")
    gidx = torch.empty((B, n), dtype=torch.int32, device=gm.device)
    counts = torch.empty((B,), dtype=torch.int32, device=gm.device)
    _lib.check(_lib.lib().lf_global_index(_ptr(gm), B, n, _ptr(gidx), _ptr(counts),
                                          _stream_ptr(stream)), "lf_global_index")
    return gidx, counts


def default_max_global(global_mask) -> int:
    """Upper bound of global tokens per batch read from the mask (syncs)."""
    if global_mask is None:
        return 0
    return int((global_mask != 0).sum(dim=1).max().item())


def attention_prepare(local_mask, global_mask, *, B, H, n, max_global, workspace, stream=None):
    lm = _mask(local_mask, B, n, "local_mask")
    gm = _mask(global_mask, B, n, "global_mask")
    _dev(workspace, "workspace")
    _lib.check(_lib.lib().lf_attention_prepare(B, H, n, D_HEAD, _ptr(lm), _ptr(gm), max_global,
                                               _ptr(workspace), workspace.numel(),
                                               _stream_ptr(stream)), "lf_attention_prepare")


def attention_run(q, k, v, qg, kg, vg, *, window, dilation=None, causal=False, max_global,
                  workspace, out=None, stream=None):
    dt, (B, H, n, _) = _check_projections([q, k, v, qg, kg, vg])
    if out is None:
        out = torch.empty_like(q)
    _check_projections([q, out])
    _dev(workspace, "workspace")
    _lib.check(_lib.lib().lf_attention_run(dt, B, H, n, D_HEAD, _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(qg), _ptr(kg), _ptr(vg), max_global, int(window),
                                           _dilation(dilation, H), int(bool(causal)), _ptr(out),
                                           _ptr(workspace), workspace.numel(),
                                           _stream_ptr(stream)), "lf_attention_run")
    return out


def attention_forward(q, k, v, qg, kg, vg, local_mask=None, global_mask=None, *, window,
                      dilation=None, causal=False, max_global=None, out=None, workspace=None,
                      lse=None, stream=None):
    """Longformer attention forward; returns out [B, H, n, 64] in the input dtype.

    max_global: host upper bound on the global tokens of any batch; when None
    it is read from global_mask (one device-to-host sync).
    lse: optional fp32 [B, H, n] tensor (bf16 / fp16 only): receives each
    valid non-global row's log-sum-exp (log2 units) for attention_backward.
    """
    dt, (B, H, n, _) = _check_projections([q, k, v, qg, kg, vg])
    lm = _mask(local_mask, B, n, "local_mask")
    gm = _mask(global_mask, B, n, "global_mask")
    if max_global is None:
        max_global = default_max_global(gm)
    if workspace is None:
        workspace = new_workspace(B, H, n, max_global, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check_projections([q, out])
    _dev(workspace, "workspace")
    if lse is not None:
        _check_lse(lse, B, H, n, q.device)
        _lib.check(_lib.lib().lf_attention_forward_lse(
            dt, B, H, n, D_HEAD, _ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg), _ptr(vg),
            _ptr(lm), _ptr(gm), int(max_global), int(window), _dilation(dilation, H),
            int(bool(causal)), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
            _stream_ptr(stream)), "lf_attention_forward_lse")
        return out
    _lib.check(_lib.lib().lf_attention_forward(
        dt, B, H, n, D_HEAD, _ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg), _ptr(vg), _ptr(lm),
        _ptr(gm), int(max_global), int(window), _dilation(dilation, H), int(bool(causal)),
        _ptr(out), _ptr(workspace), workspace.numel(), _stream_ptr(stream)),
        "lf_attention_forward")
    return out


def _check_lse(lse, B, H, n, device):
    if (not isinstance(lse, torch.Tensor) or lse.dtype != torch.float32
            or tuple(lse.shape) != (B, H, n) or not lse.is_contiguous() or lse.device != device):
        raise ValueError("lse must be a contiguous fp32 [B, H, n] tensor on the inputs' device")


def host_staging_size(dtype: torch.dtype, B: int, H: int, n: int) -> int:
    return int(_lib.lib().lf_host_staging_size(_DTYPES[dtype], B, H, n, D_HEAD))


def host_copy_bytes(dtype: torch.dtype, B: int, H: int, n: int, local_mask=None,
                    global_mask=None) -> int:
    """Host-to-device bytes attention_forward_host copies for these host masks
    (only what the kernels read; see lf_host_copy_bytes)."""
    for m in (local_mask, global_mask):
        if m is not None and (m.is_cuda or m.dtype not in (torch.uint8, torch.bool)
                              or tuple(m.shape) != (B, n) or not m.is_contiguous()):
            raise ValueError("host masks must be contiguous uint8 CPU tensors of shape [B, n]")
    return int(_lib.lib().lf_host_copy_bytes(_DTYPES[dtype], B, H, n, D_HEAD, _ptr(local_mask),
                                             _ptr(global_mask)))


def attention_forward_host(q, k, v, qg, kg, vg, local_mask=None, global_mask=None, *, window,
                           dilation=None, causal=False, max_global, out, staging, workspace,
                           stream=None):
    """The whole forward from host (ideally pinned) tensors: copies in, runs,
    copies the output back into the host tensor ``out`` and synchronises."""
    q0 = q
    if q0.dtype not in _DTYPES or q0.dim() != 4 or q0.shape[-1] != D_HEAD:
        raise ValueError("projections must be [B, H, n, 64] of a supported dtype")
    B, H, n, _ = q0.shape
    for t in (k, v, qg, kg, vg, out):
        if t.is_cuda or t.shape != q0.shape or t.dtype != q0.dtype or not t.is_contiguous():
            raise ValueError("host tensors must be contiguous CPU tensors of one shape/dtype")
    for m in (local_mask, global_mask):
        if m is not None and (m.is_cuda or m.dtype not in (torch.uint8, torch.bool)
                              or tuple(m.shape) != (B, n) or not m.is_contiguous()):
            raise ValueError("host masks must be contiguous uint8 CPU tensors of shape [B, n]")
    _dev(staging, "staging")
    _dev(workspace, "workspace")
    rc = _lib.lib().lf_attention_forward_host(
        _DTYPES[q0.dtype], B, H, n, D_HEAD, _ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg),
        _ptr(vg), _ptr(local_mask), _ptr(global_mask), int(max_global), int(window),
        _dilation(dilation, H), int(bool(causal)), _ptr(out), _ptr(staging), staging.numel(),
        _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    _lib.check(rc, "lf_attention_forward_host")
    return out


def workspace_status(workspace, stream=None) -> int:
    """Synchronises the stream and returns the device status word."""
    _dev(workspace, "workspace")
    return int(_lib.lib().lf_workspace_status(_ptr(workspace), _stream_ptr(stream)))


def attention_forward_static(q, k, v, qg, kg, vg, local_mask=None, global_mask=None, *, window,
                             dilation=None, causal=False, max_global, out, stream=None) -> int:
    """``lf_attention_forward_static``: the forward with its workspace in the
    library's fixed per-device scratch (no device allocation by the call).

    ``out`` and ``max_global`` are required, so the binding allocates nothing
    either.  Returns the device address of the scratch, for
    ``scratch_status``.  Calls on one device must not overlap in time.
    """
    dt, (B, H, n, _) = _check_projections([q, k, v, qg, kg, vg])
    _check_projections([q, out])
    lm = _mask(local_mask, B, n, "local_mask")
    gm = _mask(global_mask, B, n, "global_mask")
    scratch = ctypes.c_void_p()
    _lib.check(_lib.lib().lf_attention_forward_static(
        dt, B, H, n, D_HEAD, _ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg), _ptr(vg), _ptr(lm),
        _ptr(gm), int(max_global), int(window), _dilation(dilation, H), int(bool(causal)),
        _ptr(out), _stream_ptr(stream), ctypes.byref(scratch)),
        "lf_attention_forward_static")
    return int(scratch.value)


def scratch_status(scratch: int, stream=None) -> int:
    """Synchronises the stream and returns the status word of the last
    ``attention_forward_static`` call that used ``scratch``."""
    return int(_lib.lib().lf_workspace_status(ctypes.c_void_p(scratch), _stream_ptr(stream)))


def qkv_projection(x, w, bias=None, wqg=None, bqg=None, global_idx=None, counts=None, *,
                   H: int, max_global: int = 0, out=None, status=None, stream=None):
    """``lf_qkv_projection``: Q, K, V, Kg, Vg of every token and Qg of the
    global tokens, each [B, H, n, 64] in x's dtype.

    x [B, n, H*64]; w [5*H*64, H*64] (Q, K, V, Kg, Vg stacked, rows = output
    features); bias [5*H*64] or None; wqg [H*64, H*64] and bqg [H*64] for Qg
    (skipped when wqg is None or max_global is 0); global_idx [B, n] and
    counts [B] int32 as from ``global_index``.  ``out`` may hold preallocated
    tensors under the keys q, k, v, qg, kg, vg.  Qg rows at non-global
    positions are left as they are (zeros when this call allocates qg).
    """
    if x.dtype not in (torch.bfloat16, torch.float16) or x.dim() != 3:
        raise ValueError("x must be a [B, n, H*64] bf16 or fp16 CUDA tensor")
    B, n, hid = x.shape
    if hid != H * D_HEAD:
        raise ValueError("x's last dimension must be H * 64")
    for t in (x, w, bias, wqg, bqg):
        if t is not None and (not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype):
            raise ValueError("x, w, bias, wqg, bqg must be contiguous CUDA tensors of one dtype")
    _dev(w, "w", x.dtype, (5 * hid, hid))
    _dev(bias, "bias", x.dtype, (5 * hid,))
    _dev(wqg, "wqg", x.dtype, (hid, hid))
    _dev(bqg, "bqg", x.dtype, (hid,))
    outs = dict(out or {})
    for name in ("q", "k", "v", "kg", "vg"):
        if name not in outs:
            outs[name] = torch.empty((B, H, n, D_HEAD), dtype=x.dtype, device=x.device)
    if "qg" not in outs:
        outs["qg"] = torch.zeros((B, H, n, D_HEAD), dtype=x.dtype, device=x.device)
    _check_projections([outs[k] for k in ("q", "k", "v", "qg", "kg", "vg")])
    if tuple(outs["q"].shape) != (B, H, n, D_HEAD) or outs["q"].dtype != x.dtype:
        raise ValueError("outputs must be [B, H, n, 64] in x's dtype")
    _dev(global_idx, "global_idx", torch.int32, (B, n))
    _dev(counts, "counts", torch.int32, (B,))
    _dev(status, "status", torch.int32)
    _lib.check(_lib.lib().lf_qkv_projection(
        _DTYPES[x.dtype], B, n, H, D_HEAD, _ptr(x), _ptr(w), _ptr(bias), _ptr(wqg), _ptr(bqg),
        _ptr(global_idx), _ptr(counts), int(max_global), _ptr(outs["q"]), _ptr(outs["k"]),
        _ptr(outs["v"]), _ptr(outs["qg"]), _ptr(outs["kg"]), _ptr(outs["vg"]), _ptr(status),
        _stream_ptr(stream)), "lf_qkv_projection")
    return outs


def output_workspace_size(B: int, n: int, H: int) -> int:
    return int(_lib.lib().lf_output_workspace_size(B, n, H, D_HEAD))


def output_layer(attn, wo, bo, residual, gamma, beta, *, eps: float = 1e-5, out=None,
                 workspace=None, status=None, stream=None):
    """``lf_output_layer``: LayerNorm(concat_heads(attn) . wo^T + bo + residual)
    with gamma, beta; returns out [B, n, H*64] in attn's dtype."""
    if attn.dtype not in (torch.bfloat16, torch.float16) or attn.dim() != 4 \
            or attn.shape[-1] != D_HEAD:
        raise ValueError("attn must be a [B, H, n, 64] bf16 or fp16 CUDA tensor")
    B, H, n, _ = attn.shape
    for t in (attn, wo, bo, residual, gamma, beta):
        if t is not None and (not t.is_cuda or not t.is_contiguous() or t.dtype != attn.dtype):
            raise ValueError("all inputs must be contiguous CUDA tensors of attn's dtype")
    hid = H * D_HEAD
    _dev(wo, "wo", attn.dtype, (hid, hid))
    _dev(bo, "bo", attn.dtype, (hid,))
    _dev(residual, "residual", attn.dtype, (B, n, hid))
    _dev(gamma, "gamma", attn.dtype, (hid,))
    _dev(beta, "beta", attn.dtype, (hid,))
    if out is None:
        out = torch.empty_like(residual)
    _dev(out, "out", attn.dtype, (B, n, hid))
    if workspace is None:
        workspace = torch.empty(output_workspace_size(B, n, H), dtype=torch.uint8,
                                device=attn.device)
    _dev(workspace, "workspace")
    _dev(status, "status", torch.int32)
    _lib.check(_lib.lib().lf_output_layer(
        _DTYPES[attn.dtype], B, n, H, D_HEAD, _ptr(attn), _ptr(wo), _ptr(bo), _ptr(residual),
        _ptr(gamma), _ptr(beta), float(eps), _ptr(out), _ptr(workspace), workspace.numel(),
        _ptr(status), _stream_ptr(stream)), "lf_output_layer")
    return out


def backward_scratch_size(B: int, H: int, n: int, max_global: int) -> int:
    return int(_lib.lib().lf_backward_scratch_size(B, H, n, D_HEAD, max_global))


def attention_backward(q, k, v, qg, kg, vg, out, dout, *, window, dilation=None, causal=False,
                       max_global, workspace, grads=None, scratch=None, lse=None, stream=None):
    """``lf_attention_backward``: gradients of the attention with respect to
    q, k, v, qg, kg, vg given the forward output ``out`` and dLoss/dout.

    ``workspace`` is the forward's prepared workspace (same masks and
    max_global).  ``lse``: the log-sum-exp attention_forward(lse=...) wrote
    for these inputs (bf16 / fp16), read instead of recomputed.  Returns a
    dict of the six gradients (``grads`` may supply them, keyed q, k, v, qg,
    kg, vg).
    """
    dt, (B, H, n, _) = _check_projections([q, k, v, qg, kg, vg])
    _check_projections([q, out, dout])
    names = ("q", "k", "v", "qg", "kg", "vg")
    if grads is None:
        grads = {nm: torch.empty_like(q) for nm in names}
    _check_projections([q] + [grads[nm] for nm in names])
    if scratch is None:
        scratch = torch.empty(backward_scratch_size(B, H, n, max_global), dtype=torch.uint8,
                              device=q.device)
    _dev(workspace, "workspace")
    _dev(scratch, "scratch")
    if lse is not None:
        _check_lse(lse, B, H, n, q.device)
        _lib.check(_lib.lib().lf_attention_backward_lse(
            dt, B, H, n, D_HEAD, _ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg), _ptr(vg),
            _ptr(out), _ptr(dout), _ptr(lse), int(max_global), int(window),
            _dilation(dilation, H), int(bool(causal)), *[_ptr(grads[nm]) for nm in names],
            _ptr(workspace), workspace.numel(), _ptr(scratch), scratch.numel(),
            _stream_ptr(stream)), "lf_attention_backward_lse")
        return grads
    _lib.check(_lib.lib().lf_attention_backward(
        dt, B, H, n, D_HEAD, _ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg), _ptr(vg), _ptr(out),
        _ptr(dout), int(max_global), int(window), _dilation(dilation, H), int(bool(causal)),
        *[_ptr(grads[nm]) for nm in names], _ptr(workspace), workspace.numel(), _ptr(scratch),
        scratch.numel(), _stream_ptr(stream)), "lf_attention_backward")
    return grads


def ffn_workspace_size(B: int, n: int, hidden: int, inter: int) -> int:
    return int(_lib.lib().lf_ffn_workspace_size(B, n, hidden, inter))


def ffn_block(h, w1, b1, w2, b2, gamma, beta, *, eps: float = 1e-5, out=None, workspace=None,
              status=None, stream=None):
    """``lf_ffn_block``: LayerNorm(GELU(h w1^T + b1) w2^T + b2 + h) with gamma,
    beta; h [B, n, hidden] bf16 / fp16; returns out [B, n, hidden]."""
    if h.dtype not in (torch.bfloat16, torch.float16) or h.dim() != 3:
        raise ValueError("h must be a [B, n, hidden] bf16 or fp16 CUDA tensor")
    B, n, hidden = h.shape
    inter = w1.shape[0]
    for t in (h, w1, b1, w2, b2, gamma, beta):
        if t is not None and (not t.is_cuda or not t.is_contiguous() or t.dtype != h.dtype):
            raise ValueError("all inputs must be contiguous CUDA tensors of h's dtype")
    if tuple(w1.shape) != (inter, hidden) or tuple(w2.shape) != (hidden, inter):
        raise ValueError("w1 must be [inter, hidden] and w2 [hidden, inter]")
    _dev(b1, "b1", h.dtype, (inter,))
    _dev(b2, "b2", h.dtype, (hidden,))
    _dev(gamma, "gamma", h.dtype, (hidden,))
    _dev(beta, "beta", h.dtype, (hidden,))
    if out is None:
        out = torch.empty_like(h)
    _dev(out, "out", h.dtype, (B, n, hidden))
    if workspace is None:
        workspace = torch.empty(max(1, ffn_workspace_size(B, n, hidden, inter)),
                                dtype=torch.uint8, device=h.device)
    _dev(workspace, "workspace")
    _dev(status, "status", torch.int32)
    _lib.check(_lib.lib().lf_ffn_block(
        _DTYPES[h.dtype], B, n, hidden, inter, _ptr(h), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2),
        _ptr(gamma), _ptr(beta), float(eps), _ptr(out), _ptr(workspace), workspace.numel(),
        _ptr(status), _stream_ptr(stream)), "lf_ffn_block")
    return out


def encoder_workspace_size(B: int, n: int, H: int, inter: int, max_global: int) -> int:
    return int(_lib.lib().lf_encoder_workspace_size(B, n, H, D_HEAD, inter, max_global))


def encoder_forward(x, layers, local_mask=None, global_mask=None, *, H: int, windows,
                    dilations=None, max_global=None, eps: float = 1e-5, out=None,
                    workspace=None, stream=None):
    """``lf_encoder_forward``: a stack of Longformer encoder layers.

    x [B, n, H*64] bf16 / fp16; layers: a list of dicts of CUDA tensors keyed
    like ``lf_layer_weights`` (w_qkv, b_qkv, w_qg, b_qg, w_o, b_o, ln1_gamma,
    ln1_beta, w_1, b_1, w_2, b_2, ln2_gamma, ln2_beta; biases and w_qg may be
    missing or None); windows: one per layer; dilations: None or one list of H
    values per layer.
    """
    if x.dtype not in (torch.bfloat16, torch.float16) or x.dim() != 3:
        raise ValueError("x must be a [B, n, H*64] bf16 or fp16 CUDA tensor")
    B, n, hid = x.shape
    if hid != H * D_HEAD:
        raise ValueError("x's last dimension must be H*64")
    _dev(x, "x")
    L = len(layers)
    if len(windows) != L or (dilations is not None and len(dilations) != L):
        raise ValueError("windows (and dilations) need one entry per layer")
    inter = layers[0]["w_1"].shape[0]
    arr = (_lib.LayerWeights * L)()
    for i, lw in enumerate(layers):
        for f in _lib.LAYER_FIELDS:
            t = lw.get(f)
            if t is not None:
                if not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype:
                    raise ValueError(f"layer {i} {f}: must be a contiguous CUDA tensor of "
                                     "x's dtype")
                setattr(arr[i], f, t.data_ptr())
        if lw["w_1"].shape[0] != inter:
            raise ValueError("all layers must share the intermediate size")
        shapes = {"w_qkv": (5 * hid, hid), "b_qkv": (5 * hid,), "w_qg": (hid, hid),
                  "b_qg": (hid,), "w_o": (hid, hid), "b_o": (hid,), "ln1_gamma": (hid,),
                  "ln1_beta": (hid,), "w_1": (inter, hid), "b_1": (inter,), "w_2": (hid, inter),
                  "b_2": (hid,), "ln2_gamma": (hid,), "ln2_beta": (hid,)}
        for f, shp in shapes.items():
            _dev(lw.get(f), f"layer {i} {f}", x.dtype, shp)
    lm = _mask(local_mask, B, n, "local_mask")
    gm = _mask(global_mask, B, n, "global_mask")
    if max_global is None:
        max_global = default_max_global(gm)
    win = (ctypes.c_int32 * L)(*[int(w) for w in windows])
    dil = None
    if dilations is not None:
        flat = []
        for dl in dilations:
            vals = [1] * H if dl is None else [int(v) for v in dl]
            if len(vals) != H:
                raise ValueError("each layer's dilation needs H entries")
            flat += vals
        dil = (ctypes.c_int32 * (L * H))(*flat)
    if out is None:
        out = torch.empty_like(x)
    _dev(out, "out", x.dtype, (B, n, hid))
    if workspace is None:
        workspace = torch.empty(max(1, encoder_workspace_size(B, n, H, inter, max_global)),
                                dtype=torch.uint8, device=x.device)
    _dev(workspace, "workspace")
    _lib.check(_lib.lib().lf_encoder_forward(
        _DTYPES[x.dtype], B, n, H, D_HEAD, inter, L, arr, win, dil, _ptr(x), _ptr(lm), _ptr(gm),
        int(max_global), float(eps), _ptr(out), _ptr(workspace), workspace.numel(),
        _stream_ptr(stream)), "lf_encoder_forward")
    return out

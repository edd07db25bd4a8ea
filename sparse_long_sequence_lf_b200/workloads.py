"""Seeded synthetic inputs for the Longformer attention forward.

This module only draws numbers and builds masks.  It holds none of the
method's arithmetic, so both the CUDA path and the fp64 oracle can take their
inputs from it without sharing any computation.

Recipe (every workload):
  * ``torch.Generator('cpu').manual_seed(seed)``; six ``randn`` fp32 tensors of
    shape [B, H, n, 64] drawn in the order Q, K, V, Qg, Kg, Vg, then cast to
    the workload dtype on the host.  Both sides see the same rounded values;
    the oracle upcasts them exactly to fp64.
  * masks are uint8 [B, n]: local mask 1 = valid, 0 = padding; global mask
    1 = global token.
  * random global positions come from ``numpy.random.default_rng(seed)``,
    drawn uniformly without replacement and sorted.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np
import torch

D_HEAD = 64

_TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" | "f16" | "bf16"
    B: int
    H: int
    n: int
    window: int
    dilation: tuple = ()  # one entry per head; empty = all 1
    causal: bool = False
    globals_kind: str = "none"   # "none" | "first:<g>" | "random:<g>" | "list:<p,p,...>"
    pad_tail: tuple = ()  # per batch: number of padded positions at the end
    seed: int = 0
    d: int = D_HEAD
    notes: str = field(default="", compare=False)

    @property
    def torch_dtype(self):
        return _TORCH_DTYPES[self.dtype]

    def dilation_list(self):
        return list(self.dilation) if self.dilation else [1] * self.H

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the measurement plan.  Their shapes follow the
# Longformer-base encoder (12 heads, n = 4096, w = 512), the QA setting of the
# FasterTransformer guide (question tokens global at the front, padded tail),
# the autoregressive dilated-window setting of the Longformer notes, and a
# long-document case with scattered global tokens.
WORKLOADS = {
    w.name: w for w in [
        Workload("fp32-b1h2-n512-w64-g1", "f32", 1, 2, 512, 64,
                 globals_kind="first:1", seed=1001),
        Workload("bf16-b1h12-n4096-w512-g1", "bf16", 1, 12, 4096, 512,
                 globals_kind="first:1", seed=1002),
        Workload("fp16-b2h16-n4096-w512-g64-pad300", "f16", 2, 16, 4096, 512,
                 globals_kind="first:64", pad_tail=(0, 300), seed=1003),
        Workload("bf16-b1h8-n8192-causal256-dil1x6-2-3", "bf16", 1, 8, 8192, 256,
                 dilation=(1, 1, 1, 1, 1, 1, 2, 3), causal=True, seed=1004),
        Workload("bf16-b1h16-n16384-w512-g32rand", "bf16", 1, 16, 16384, 512,
                 globals_kind="random:32", seed=1005),
    ]
}

# The workload the headline throughput is quoted on (Longformer-base shape).
HEADLINE = "bf16-b1h12-n4096-w512-g1"


def global_positions(wl: Workload) -> list[list[int]]:
    """Global token positions per batch (sorted, unique)."""
    kind = wl.globals_kind
    if kind == "none":
        return [[] for _ in range(wl.B)]
    tag, _, arg = kind.partition(":")
    if tag == "first":
        g = int(arg)
        return [list(range(min(g, wl.n))) for _ in range(wl.B)]
    if tag == "random":
        g = int(arg)
        rng = np.random.default_rng(wl.seed)
        pos = sorted(int(p) for p in rng.choice(wl.n, size=min(g, wl.n), replace=False))
        return [list(pos) for _ in range(wl.B)]
    if tag == "list":
        per_batch = [sorted({int(p) for p in part.split(",") if p != ""})
                     for part in arg.split(";")]
        if len(per_batch) == 1:
            per_batch = per_batch * wl.B
        return per_batch
    raise ValueError(f"unknown globals kind {kind!r}")


def make_masks(wl: Workload):
    """uint8 [B, n] local mask (1 valid) and global mask (1 global), or None."""
    local = None
    if any(wl.pad_tail):
        local = torch.ones((wl.B, wl.n), dtype=torch.uint8)
        for b, p in enumerate(wl.pad_tail):
            if p > 0:
                local[b, wl.n - p:] = 0
    glob = None
    pos = global_positions(wl)
    if any(len(p) for p in pos):
        glob = torch.zeros((wl.B, wl.n), dtype=torch.uint8)
        for b, ps in enumerate(pos):
            if ps:
                glob[b, torch.tensor(ps, dtype=torch.long)] = 1
    return local, glob


def make_projections(wl: Workload, seed: int | None = None):
    """Q, K, V, Qg, Kg, Vg as CPU tensors of the workload dtype."""
    gen = torch.Generator("cpu")
    gen.manual_seed(wl.seed if seed is None else seed)
    shape = (wl.B, wl.H, wl.n, wl.d)
    out = []
    for _ in range(6):
        t = torch.randn(shape, generator=gen, dtype=torch.float32)
        out.append(t.to(wl.torch_dtype))
    return tuple(out)


def make_inputs(wl: Workload, seed: int | None = None) -> dict:
    q, k, v, qg, kg, vg = make_projections(wl, seed)
    local, glob = make_masks(wl)
    return dict(q=q, k=k, v=v, qg=qg, kg=kg, vg=vg, local_mask=local, global_mask=glob,
                window=wl.window, dilation=wl.dilation_list(), causal=wl.causal)


def random_workload(rng: np.random.Generator, *, dtype: str = "bf16", max_n: int = 1024,
                    name: str = "random") -> Workload:
    """A small random case for parity sweeps: ragged n, random window,
    dilation, causality, global positions and tail padding."""
    B = int(rng.integers(1, 3))
    H = int(rng.integers(1, 4))
    n = int(rng.integers(1, max_n + 1))
    causal = bool(rng.random() < 0.3)
    if causal:
        window = int(rng.integers(1, 300))
    else:
        window = 2 * int(rng.integers(1, 300))
    # Mostly small dilations; one draw in four takes them up to 12, so that the
    # heads' (dilation, residue) classes can outgrow the residue tensor maps.
    dil_hi = 13 if rng.random() < 0.25 else 4
    dil = tuple(int(x) for x in rng.integers(1, dil_hi, size=H))
    if causal:
        gk = "none"
    else:
        g = int(rng.integers(0, min(n, 80) + 1))
        if g == 0:
            gk = "none"
        else:
            per_b = []
            for _ in range(B):
                ps = sorted(int(p) for p in rng.choice(n, size=g, replace=False))
                per_b.append(",".join(str(p) for p in ps))
            gk = "list:" + ";".join(per_b)
    pad = tuple(int(rng.integers(0, n // 2 + 1)) if rng.random() < 0.5 else 0 for _ in range(B))
    return Workload(name, dtype, B, H, n, window, dilation=dil, causal=causal,
                    globals_kind=gk, pad_tail=pad, seed=int(rng.integers(0, 2**31 - 1)))


def make_layer_inputs(wl: Workload, seed: int | None = None) -> dict:
    """Inputs of the projection prologue for the workload's shape: hidden
    states x [B, n, H*d] ~ N(0, 1); stacked weights w [5*H*d, H*d] and the
    global-query weights wqg [H*d, H*d] ~ N(0, 1/(H*d)) (unit-scale outputs);
    biases ~ N(0, 0.1^2); plus the workload's masks.  CPU tensors of the
    workload dtype, drawn in that order from one seeded generator."""
    gen = torch.Generator("cpu")
    gen.manual_seed((wl.seed if seed is None else seed) + 500009)
    hid = wl.H * wl.d
    scale = 1.0 / np.sqrt(hid)
    x = torch.randn((wl.B, wl.n, hid), generator=gen)
    w = torch.randn((5 * hid, hid), generator=gen) * scale
    bias = torch.randn((5 * hid,), generator=gen) * 0.1
    wqg = torch.randn((hid, hid), generator=gen) * scale
    bqg = torch.randn((hid,), generator=gen) * 0.1
    local, glob = make_masks(wl)
    dt = wl.torch_dtype
    return dict(x=x.to(dt), w=w.to(dt), bias=bias.to(dt), wqg=wqg.to(dt), bqg=bqg.to(dt),
                local_mask=local, global_mask=glob)


def make_output_inputs(wl: Workload, seed: int | None = None) -> dict:
    """Inputs of the output layer for the workload's shape: attention output
    attn [B, H, n, d] ~ N(0, 1); wo [H*d, H*d] ~ N(0, 1/(H*d)); bo ~ N(0, 0.1^2);
    residual [B, n, H*d] ~ N(0, 1); gamma ~ 1 + N(0, 0.1^2); beta ~ N(0, 0.1^2).
    CPU tensors of the workload dtype, drawn in that order."""
    gen = torch.Generator("cpu")
    gen.manual_seed((wl.seed if seed is None else seed) + 700001)
    hid = wl.H * wl.d
    attn = torch.randn((wl.B, wl.H, wl.n, wl.d), generator=gen)
    wo = torch.randn((hid, hid), generator=gen) / np.sqrt(hid)
    bo = torch.randn((hid,), generator=gen) * 0.1
    residual = torch.randn((wl.B, wl.n, hid), generator=gen)
    gamma = 1.0 + torch.randn((hid,), generator=gen) * 0.1
    beta = torch.randn((hid,), generator=gen) * 0.1
    dt = wl.torch_dtype
    return dict(attn=attn.to(dt), wo=wo.to(dt), bo=bo.to(dt), residual=residual.to(dt),
                gamma=gamma.to(dt), beta=beta.to(dt))


def make_output_grad(wl: Workload, seed: int | None = None) -> torch.Tensor:
    """dLoss/dO [B, H, n, d] ~ N(0, 1) for the backward pass, a CPU tensor of
    the workload dtype."""
    gen = torch.Generator("cpu")
    gen.manual_seed((wl.seed if seed is None else seed) + 900007)
    return torch.randn((wl.B, wl.H, wl.n, wl.d), generator=gen).to(wl.torch_dtype)


LAYER_FIELDS = ("w_qkv", "b_qkv", "w_qg", "b_qg", "w_o", "b_o", "ln1_gamma", "ln1_beta",
                "w_1", "b_1", "w_2", "b_2", "ln2_gamma", "ln2_beta")


def make_encoder_inputs(wl: Workload, layers: int, inter: int, seed: int | None = None):
    """Random-init weights of an encoder stack for the workload's shape and
    its input x [B, n, H*d] ~ N(0, 1): weight matrices ~ N(0, 1/fan_in),
    biases and LayerNorm shifts ~ N(0, 0.1^2), LayerNorm scales ~ 1 + N(0, 0.1^2).
    Returns (x, [dict per layer]) as CPU tensors of the workload dtype."""
    gen = torch.Generator("cpu")
    gen.manual_seed((wl.seed if seed is None else seed) + 1100009)
    hid = wl.H * wl.d
    dt = wl.torch_dtype
    rn = lambda *shape: torch.randn(shape, generator=gen)
    shapes = {"w_qkv": (5 * hid, hid), "b_qkv": (5 * hid,), "w_qg": (hid, hid), "b_qg": (hid,),
              "w_o": (hid, hid), "b_o": (hid,), "ln1_gamma": (hid,), "ln1_beta": (hid,),
              "w_1": (inter, hid), "b_1": (inter,), "w_2": (hid, inter), "b_2": (hid,),
              "ln2_gamma": (hid,), "ln2_beta": (hid,)}
    out = []
    for _ in range(layers):
        lw = {}
        for f in LAYER_FIELDS:
            t = rn(*shapes[f])
            if f.startswith("w_"):
                t = t / np.sqrt(shapes[f][1])
            elif f.endswith("gamma"):
                t = 1.0 + 0.1 * t
            else:
                t = 0.1 * t
            lw[f] = t.to(dt)
        out.append(lw)
    x = rn(wl.B, wl.n, hid).to(dt)
    return x, out


@dataclass(frozen=True)
class EncoderWorkload:
    """A stack of encoder layers on the attention workload ``attn`` (its B, H,
    n, window, globals and padding; every layer takes that window)."""
    name: str
    attn: Workload
    inter: int
    layers: int


# The model of the encoder latency table in the FasterTransformer Longformer
# Encoder guide ("performance benchmark": 16 heads of 64, intermediate 4096,
# window 512, 24 layers), at batch 1 and 4096 tokens in fp16.  The guide's
# inputs are random; the global tokens here follow its QA demo (the question
# tokens, global, at the front): 64 of them.
ENCODER_WORKLOADS = {
    e.name: e for e in [
        EncoderWorkload("fp16-b1h16-n4096-w512-i4096-l24",
                        Workload("fp16-b1h16-n4096-w512-g64", "f16", 1, 16, 4096, 512,
                                 globals_kind="first:64", seed=31), 4096, 24),
        EncoderWorkload("fp16-b8h16-n4096-w512-i4096-l24",
                        Workload("fp16-b8h16-n4096-w512-g64", "f16", 8, 16, 4096, 512,
                                 globals_kind="first:64", seed=32), 4096, 24),
    ]
}
ENCODER_HEADLINE = "fp16-b1h16-n4096-w512-i4096-l24"

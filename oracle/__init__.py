"""fp64 CPU oracle for the Longformer self-attention forward.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product library never imports,
links or executes anything in this directory, and this directory imports
nothing from the product package.

The arithmetic lives in ``lf_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only builds it with gcc on first use and marshals numpy arrays.
See ``lf_oracle.c`` for the passages each function follows and the readings
taken where the pages leave a step open.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lf_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liblf_oracle.so")
_lock = threading.Lock()
_lib_cache: dict[str, ctypes.CDLL] = {}

OK, BAD_ARG, UNSUPPORTED, NOMEM = 0, -1, -2, -3


def build(src: str = _SRC, out: str = _LIB_PATH, force: bool = False) -> str:
    """Compile the oracle with gcc (-O2 -fopenmp, strict IEEE: no fast-math)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    os.replace(tmp, out)
    return out


def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.lfo_global_index.argtypes = [P, I, I, P, P]
    lib.lfo_global_index.restype = I
    lib.lfo_forward.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, I, P, I,
                                I, I, I, I, P, I]
    lib.lfo_forward.restype = I
    lib.lfo_row_probs.argtypes = [I, I, I, I, P, P, P, P, P, P, I, P, I,
                                  I, I, I, P, P]
    lib.lfo_row_probs.restype = I
    lib.lfo_max_threads.argtypes = []
    lib.lfo_max_threads.restype = I
    return lib


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the oracle library (building it first when it is missing)."""
    with _lock:
        key = path or _LIB_PATH
        if key not in _lib_cache:
            if path is None:
                build()
            _lib_cache[key] = _declare(ctypes.CDLL(key))
        return _lib_cache[key]


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor: upcast exactly on the CPU
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _u8(a) -> np.ndarray | None:
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a != 0, dtype=np.uint8)


def _dil(dilation, H: int) -> np.ndarray | None:
    if dilation is None:
        return None
    d = np.ascontiguousarray(np.asarray(dilation, dtype=np.int32).reshape(-1))
    if d.shape[0] != H:
        raise ValueError("dilation must have one entry per head")
    return d


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__({BAD_ARG: "invalid argument", UNSUPPORTED: "unsupported",
                          NOMEM: "out of memory"}.get(code, f"error {code}"))
        self.code = code


class Oracle:
    """Thin marshalling wrapper around one loaded oracle library."""

    def __init__(self, lib: ctypes.CDLL | None = None):
        self.lib = lib if lib is not None else load()

    def global_index(self, global_mask):
        gm = _u8(global_mask)
        B, n = gm.shape
        gidx = np.empty((B, n), dtype=np.int32)
        counts = np.empty((B,), dtype=np.int32)
        rc = self.lib.lfo_global_index(_ptr(gm), B, n, _ptr(gidx), _ptr(counts))
        if rc != OK:
            raise OracleError(rc)
        return gidx, counts

    def forward(self, q, k, v, qg, kg, vg, local_mask=None, global_mask=None, *,
                window: int, dilation=None, causal: bool = False,
                bh_range=None, row_range=None, threads: int = 0, out=None):
        q, k, v, qg, kg, vg = (_f64(t) for t in (q, k, v, qg, kg, vg))
        B, H, n, d = q.shape
        for t in (k, v, qg, kg, vg):
            if t.shape != q.shape:
                raise ValueError("all six projections must have shape [B, H, n, d]")
        lm, gm = _u8(local_mask), _u8(global_mask)
        dil = _dil(dilation, H)
        bh0, bh1 = bh_range if bh_range is not None else (0, B * H)
        r0, r1 = row_range if row_range is not None else (0, n)
        if out is None:
            out = np.full((B, H, n, d), np.nan)
        rc = self.lib.lfo_forward(B, H, n, d, _ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg),
                                  _ptr(vg), _ptr(lm), _ptr(gm), int(window), _ptr(dil),
                                  int(bool(causal)), bh0, bh1, r0, r1, _ptr(out), int(threads))
        if rc != OK:
            raise OracleError(rc)
        return out

    def row_probs(self, q, k, qg, kg, local_mask=None, global_mask=None, *, window: int,
                  dilation=None, causal: bool = False, b: int = 0, h: int = 0, i: int = 0):
        q, k, qg, kg = (_f64(t) for t in (q, k, qg, kg))
        B, H, n, d = q.shape
        lm, gm = _u8(local_mask), _u8(global_mask)
        dil = _dil(dilation, H)
        cap = n + int(window) + 2
        keys = np.empty((cap,), dtype=np.int32)
        probs = np.empty((cap,), dtype=np.float64)
        rc = self.lib.lfo_row_probs(B, H, n, d, _ptr(q), _ptr(k), _ptr(qg), _ptr(kg),
                                    _ptr(lm), _ptr(gm), int(window), _ptr(dil),
                                    int(bool(causal)), b, h, i, _ptr(keys), _ptr(probs))
        if rc < 0:
            raise OracleError(rc)
        return keys[:rc].copy(), probs[:rc].copy()

    def max_threads(self) -> int:
        return int(self.lib.lfo_max_threads())


_default: Oracle | None = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def global_index(global_mask):
    return default().global_index(global_mask)


def forward(*args, **kwargs):
    return default().forward(*args, **kwargs)


def row_probs(*args, **kwargs):
    return default().row_probs(*args, **kwargs)

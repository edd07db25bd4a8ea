"""ctypes loader of the in-tree CUDA library (``_build/liblf_attention.so``).

There is no fallback: if the library is missing or fails to load, every call
raises.  Build it with ``python -m sparse_long_sequence_lf_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "_build", "liblf_attention.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "lf_attention.h")

LF_F32, LF_F16, LF_BF16 = 0, 1, 2
STATUS = {
    0: "LF_OK",
    -1: "LF_ERR_INVALID_ARG",
    -2: "LF_ERR_UNSUPPORTED",
    -3: "LF_ERR_WORKSPACE",
    -4: "LF_ERR_CUDA",
    -5: "LF_ERR_DEVICE_TIMEOUT",
    -6: "LF_ERR_GLOBAL_OVERFLOW",
    -7: "LF_ERR_NO_DEVICE",
    -8: "LF_ERR_SCRATCH_LIMIT",
}
STATIC_SCRATCH_BYTES = 16 * 1024 * 1024

_lock = threading.Lock()
_lib: ctypes.CDLL | None = None


class LfError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        name = STATUS.get(code, f"status {code}")
        super().__init__(f"{what}: {name}" if what else name)
        self.code = code
        self.name = name


def header_symbols() -> list[str]:
    """Names of the entry points declared in include/lf_attention.h."""
    text = open(HEADER).read()
    return re.findall(r"^LF_API\s+[\w\s\*]+?\b(lf_\w+)\s*\(", text, flags=re.M)


LAYER_FIELDS = ("w_qkv", "b_qkv", "w_qg", "b_qg", "w_o", "b_o", "ln1_gamma", "ln1_beta",
                "w_1", "b_1", "w_2", "b_2", "ln2_gamma", "ln2_beta")


class LayerWeights(ctypes.Structure):
    """``lf_layer_weights``: device pointers of one encoder layer."""
    _fields_ = [(f, ctypes.c_void_p) for f in LAYER_FIELDS]


def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "lf_version": (I, []),
        "lf_status_string": (ctypes.c_char_p, [I]),
        "lf_global_index": (I, [P, I, I, P, P, P]),
        "lf_workspace_size": (Z, [I, I, I, I, I]),
        "lf_attention_prepare": (I, [I, I, I, I, P, P, I, P, Z, P]),
        "lf_attention_run": (I, [I, I, I, I, I, P, P, P, P, P, P, I, I, P, I, P, P, Z, P]),
        "lf_attention_forward": (I, [I, I, I, I, I, P, P, P, P, P, P, P, P, I, I, P, I, P, P,
                                     Z, P]),
        "lf_host_staging_size": (Z, [I, I, I, I, I]),
        "lf_host_copy_bytes": (Z, [I, I, I, I, I, P, P]),
        "lf_attention_forward_host": (I, [I, I, I, I, I, P, P, P, P, P, P, P, P, I, I, P, I, P,
                                          P, Z, P, Z, P]),
        "lf_workspace_status": (I, [P, P]),
        "lf_test_forward_hooks": (I, [ctypes.c_ulonglong, I]),
        "lf_exp2_poly_eval": (I, [P, P, I, P]),
        "lf_attention_forward_static": (I, [I, I, I, I, I, P, P, P, P, P, P, P, P, I, I, P, I, P,
                                            P, ctypes.POINTER(P)]),
        "lf_qkv_projection": (I, [I, I, I, I, I, P, P, P, P, P, P, P, I, P, P, P, P, P, P, P, P]),
        "lf_output_workspace_size": (Z, [I, I, I, I]),
        "lf_output_layer": (I, [I, I, I, I, I, P, P, P, P, P, P, ctypes.c_float, P, P, Z, P, P]),
        "lf_ffn_workspace_size": (Z, [I, I, I, I]),
        "lf_ffn_block": (I, [I, I, I, I, I, P, P, P, P, P, P, P, ctypes.c_float, P, P, Z, P, P]),
        "lf_encoder_workspace_size": (Z, [I, I, I, I, I, I]),
        "lf_encoder_forward": (I, [I, I, I, I, I, I, I, ctypes.POINTER(LayerWeights), P, P, P, P,
                                   P, I, ctypes.c_float, P, P, Z, P]),
        "lf_backward_scratch_size": (Z, [I, I, I, I, I]),
        "lf_attention_backward": (I, [I, I, I, I, I, P, P, P, P, P, P, P, P, I, I, P, I, P, P, P,
                                      P, P, P, P, Z, P, Z, P]),
        "lf_attention_forward_lse": (I, [I, I, I, I, I, P, P, P, P, P, P, P, P, I, I, P, I, P, P,
                                         P, Z, P]),
        "lf_attention_backward_lse": (I, [I, I, I, I, I, P, P, P, P, P, P, P, P, P, I, I, P, I, P,
                                          P, P, P, P, P, P, Z, P, Z, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"CUDA library not built: {LIB_PATH} is missing "
                    "(run python -m sparse_long_sequence_lf_b200.build)")
            _lib = _declare(ctypes.CDLL(LIB_PATH))
        return _lib


def check(code: int, what: str = "") -> None:
    if code != 0:
        raise LfError(code, what)

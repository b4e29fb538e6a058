"""ctypes binding of libattn.so (argument marshalling only; every step runs in the CUDA
kernels behind the C-ABI declared in include/attn.h)."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")

ATTN_OK = 0
ATTN_ERR_INVALID = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_CUDA = -3
ATTN_ERR_TIMEOUT = -4
ATTN_ERR_NOMEM = -5
ATTN_ERR_CHECK = -6

MASK_NONE = 0
MASK_CAUSAL = 1
MASK_WINDOW = 2
MASK_DOC = 4

# Every symbol include/attn.h declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
SIGNATURES = {
    "attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _F, _P, _P, _P]),
    "attn_fwd_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _F, _P, _P, _P]),
    "attn_fwd_gqa": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _F, _P, _P, _P]),
    "attn_fwd_pair": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _F, _P, _P, _P]),
    "attn_fwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _F,
                             _P, _P]),
    "attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _F, _P, _P, _P]),
    "attn_tile_map_build": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "attn_fwd_with_map": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _F, _P, _P, _P, _P, _P]),
    "attn_quantize_e4m3": (_I, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "attn_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _F, _P, _P, _P]),
    "attn_quantize_mxfp4": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "attn_fwd_fp4": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "attn_get_status": (_I, [_P]),
    "attn_strerror": (ctypes.c_char_p, [_I]),
    "attn_shutdown": (None, []),
    "attn_debug_set_fault": (None, [_I, _I]),
}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


def open_library(path: str) -> ctypes.CDLL:
    """Opens a build of libattn.so at ``path`` with the ctypes signatures of include/attn.h."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing; build it with `python -m tiled_attention_14_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load() -> ctypes.CDLL:
    """Loads the in-tree libattn.so (raises if it is missing: there is no fallback).  The
    environment variable TILED_ATTENTION_LIB may name another build of the same sources
    (the ablation builds) for measurements."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = open_library(os.environ.get("TILED_ATTENTION_LIB") or LIB_PATH)
    return _lib


def strerror(code: int) -> str:
    return load().attn_strerror(code).decode()


def check(code: int, what: str) -> None:
    if code != ATTN_OK:
        raise AttnError(code, what)

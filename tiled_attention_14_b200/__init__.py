"""B200-native fused attention forward (sm_100a): the Python face of libattn.so.

Each function takes torch CUDA tensors, passes their device pointers and the current
CUDA stream to the C-ABI (include/attn.h) and raises ``AttnError`` on a nonzero status.
PyTorch serves only for device memory and streams; there is no CPU path.
"""
from __future__ import annotations

import math

import torch

from ._lib import (ATTN_ERR_TIMEOUT, ATTN_OK, MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW,
                   AttnError, check, load)

__all__ = ["attn_fwd", "attn_fwd_noalloc", "attn_fwd_with_map", "attn_fwd_fp8", "attn_quantize_e4m3",
           "attn_tile_map_build", "attn_get_status", "attn_shutdown", "tile_map_shape",
           "AttnError", "MASK_NONE", "MASK_CAUSAL", "MASK_WINDOW", "MASK_DOC"]


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _out(q, o, lse):
    B, H, Sq, D = q.shape
    if o is None:
        o = torch.empty(B, H, Sq, D, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(B, H, Sq, dtype=torch.float32, device=q.device)
    return o, lse


def attn_fwd(q, k, v, o=None, lse=None, scale=None, mask_kind=MASK_NONE, window=0, softcap=0.0,
             alibi_slopes=None, doc_ids=None, stream=None):
    """BF16 attention forward. q [B,H,Sq,D], k/v [B,H,Sk,D] bf16 contiguous on one device.
    Returns (o bf16 [B,H,Sq,D], lse fp32 [B,H,Sq])."""
    lib = load()
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    o, lse = _out(q, o, lse)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Sq, Sk, D, float(scale),
                      int(mask_kind), int(window), float(softcap), _ptr(alibi_slopes), _ptr(doc_ids),
                      _stream(stream))
    check(rc, "attn_fwd")
    return o, lse


def attn_fwd_noalloc(q, k, v, o, lse, scale=None, mask_kind=MASK_NONE, window=0, softcap=0.0,
                     alibi_slopes=None, doc_ids=None, stream=None):
    """attn_fwd without any device allocation inside the call: the caller passes the
    outputs, and the document-mask tile map uses the library's fixed per-device array
    (see include/attn.h).  For callers that cannot allocate during the call."""
    lib = load()
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = lib.attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Sq, Sk, D, float(scale),
                              int(mask_kind), int(window), float(softcap), _ptr(alibi_slopes), _ptr(doc_ids),
                              _stream(stream))
    check(rc, "attn_fwd_noalloc")
    return o, lse


def tile_map_shape(B, Sq, Sk):
    return (B, (Sq + 255) // 256), (B, (Sq + 255) // 256, (Sk + 127) // 128)


def attn_tile_map_build(B, Sq, Sk, mask_kind, window=0, doc_ids=None, device=None, stream=None):
    """Returns (counts int32 [B, nqb], entries int32 view of uint32 [B, nqb, nkt])."""
    lib = load()
    device = device if device is not None else (doc_ids.device if doc_ids is not None else "cuda")
    cs, es = tile_map_shape(B, Sq, Sk)
    counts = torch.empty(cs, dtype=torch.int32, device=device)
    entries = torch.zeros(es, dtype=torch.int32, device=device)
    rc = lib.attn_tile_map_build(_ptr(counts), _ptr(entries), B, Sq, Sk, int(mask_kind), int(window),
                                 _ptr(doc_ids), _stream(stream))
    check(rc, "attn_tile_map_build")
    return counts, entries


def attn_fwd_with_map(q, k, v, counts, entries, o=None, lse=None, scale=None, mask_kind=MASK_NONE,
                      window=0, softcap=0.0, alibi_slopes=None, doc_ids=None, stream=None):
    lib = load()
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    o, lse = _out(q, o, lse)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = lib.attn_fwd_with_map(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Sq, Sk, D,
                               float(scale), int(mask_kind), int(window), float(softcap),
                               _ptr(alibi_slopes), _ptr(doc_ids), _ptr(counts), _ptr(entries),
                               _stream(stream))
    check(rc, "attn_fwd_with_map")
    return o, lse


def attn_quantize_e4m3(x, xq=None, scales=None, stream=None):
    """fp32 [B,H,S,D] -> (e4m3 codes uint8 [B,H,S,D], fp32 scales [B,H,ceil(S/128)])."""
    lib = load()
    B, H, S, D = x.shape
    if xq is None:
        xq = torch.empty(B, H, S, D, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(B, H, (S + 127) // 128, dtype=torch.float32, device=x.device)
    rc = lib.attn_quantize_e4m3(_ptr(x), _ptr(xq), _ptr(scales), B, H, S, D, _stream(stream))
    check(rc, "attn_quantize_e4m3")
    return xq, scales


def attn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o=None, lse=None, scale=None,
                 mask_kind=MASK_NONE, window=0, softcap=0.0, alibi_slopes=None, doc_ids=None,
                 stream=None):
    lib = load()
    B, H, Sq, D = q8.shape
    Sk = k8.shape[2]
    o, lse = _out(q8, o, lse)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = lib.attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
                          _ptr(o), _ptr(lse), B, H, Sq, Sk, D, float(scale), int(mask_kind), int(window),
                          float(softcap), _ptr(alibi_slopes), _ptr(doc_ids), _stream(stream))
    check(rc, "attn_fwd_fp8")
    return o, lse


def attn_get_status(stream=None) -> int:
    return load().attn_get_status(_stream(stream))


def attn_shutdown() -> None:
    load().attn_shutdown()

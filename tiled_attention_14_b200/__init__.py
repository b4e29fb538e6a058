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

__all__ = ["attn_fwd", "attn_fwd_pair", "attn_bwd", "attn_fwd_varlen", "attn_fwd_noalloc", "attn_fwd_with_map", "attn_fwd_fp8", "attn_quantize_e4m3",
           "attn_quantize_mxfp4", "attn_fwd_fp4", "mxfp4_shapes",
           "attn_tile_map_build", "attn_get_status", "attn_shutdown", "tile_map_shape",
           "AttnError", "MASK_NONE", "MASK_CAUSAL", "MASK_WINDOW", "MASK_DOC"]


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need(t, name, dtype, shape, device):
    """Raises ValueError unless ``t`` is a contiguous tensor of this dtype and shape on
    ``device``.  The C-ABI receives bare pointers and cannot check sizes itself, so a
    wrong tensor here would make a kernel read or write out of bounds."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name}: expected a torch tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _check_qkv(q, k, v, dtype, gqa=False):
    """q [B,H,Sq,D], k and v [B,H,Sk,D] (with ``gqa``: [B,Hkv,Sk,D], Hkv dividing H) of
    ``dtype``, contiguous, on one CUDA device."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q: expected a 4-d tensor [B, H, Sq, D]")
    if q.device.type != "cuda":
        raise ValueError(f"q: on {q.device}, expected a CUDA device (there is no CPU path)")
    B, H, Sq, D = q.shape
    _need(q, "q", dtype, (B, H, Sq, D), q.device)
    if not isinstance(k, torch.Tensor) or k.dim() != 4:
        raise ValueError("k: expected a 4-d tensor [B, H, Sk, D]")
    Hkv, Sk = k.shape[1], k.shape[2]
    if not gqa and Hkv != H:
        raise ValueError(f"k: {Hkv} heads, expected {H}")
    if Hkv < 1 or H % Hkv != 0:
        raise ValueError(f"k: {Hkv} key/value heads do not divide {H} query heads")
    _need(k, "k", dtype, (B, Hkv, Sk, D), q.device)
    _need(v, "v", dtype, (B, Hkv, Sk, D), q.device)
    if gqa:
        return B, H, Hkv, Sq, Sk, D
    return B, H, Sq, Sk, D


def _check_mods(q, H, B, Sk, alibi_slopes, doc_ids):
    if alibi_slopes is not None:
        _need(alibi_slopes, "alibi_slopes", torch.float32, (H,), q.device)
    if doc_ids is not None:
        _need(doc_ids, "doc_ids", torch.int32, (B, Sk), q.device)


def _out(q, o, lse):
    B, H, Sq, D = q.shape
    if o is None:
        o = torch.empty(B, H, Sq, D, dtype=torch.bfloat16, device=q.device)
    else:
        _need(o, "o", torch.bfloat16, (B, H, Sq, D), q.device)
    if lse is None:
        lse = torch.empty(B, H, Sq, dtype=torch.float32, device=q.device)
    else:
        _need(lse, "lse", torch.float32, (B, H, Sq), q.device)
    return o, lse


def attn_fwd(q, k, v, o=None, lse=None, scale=None, mask_kind=MASK_NONE, window=0, softcap=0.0,
             alibi_slopes=None, doc_ids=None, stream=None):
    """BF16 attention forward. q [B,H,Sq,D], k/v [B,Hkv,Sk,D] bf16 contiguous on one device;
    Hkv < H (dividing it) selects grouped-query heads (attn_fwd_gqa).
    Returns (o bf16 [B,H,Sq,D], lse fp32 [B,H,Sq])."""
    lib = load()
    B, H, Hkv, Sq, Sk, D = _check_qkv(q, k, v, torch.bfloat16, gqa=True)
    _check_mods(q, H, B, Sk, alibi_slopes, doc_ids)
    o, lse = _out(q, o, lse)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if Hkv == H:
        rc = lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Sq, Sk, D, float(scale),
                          int(mask_kind), int(window), float(softcap), _ptr(alibi_slopes), _ptr(doc_ids),
                          _stream(stream))
        check(rc, "attn_fwd")
    else:
        rc = lib.attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, Sq, Sk, D, float(scale),
                              int(mask_kind), int(window), float(softcap), _ptr(alibi_slopes), _ptr(doc_ids),
                              _stream(stream))
        check(rc, "attn_fwd_gqa")
    return o, lse


def attn_fwd_pair(q, k, v, o=None, lse=None, scale=None, mask_kind=MASK_NONE, window=0, softcap=0.0,
                  alibi_slopes=None, doc_ids=None, stream=None):
    """attn_fwd computed on pairs of SMs (2-CTA clusters, tcgen05 cta_group::2); BF16, D = 128.
    Same arguments and results as attn_fwd (grouped heads included); slower than attn_fwd on
    B200, kept as a tested alternative."""
    lib = load()
    B, H, Hkv, Sq, Sk, D = _check_qkv(q, k, v, torch.bfloat16, gqa=True)
    if D != 128:
        raise ValueError("attn_fwd_pair needs D = 128")
    _check_mods(q, H, B, Sk, alibi_slopes, doc_ids)
    o, lse = _out(q, o, lse)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = lib.attn_fwd_pair(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, Sq, Sk, D, float(scale),
                           int(mask_kind), int(window), float(softcap), _ptr(alibi_slopes), _ptr(doc_ids),
                           _stream(stream))
    check(rc, "attn_fwd_pair")
    return o, lse


def attn_bwd(q, k, v, o, lse, dout, dq=None, dk=None, dv=None, scale=None, mask_kind=MASK_NONE, window=0,
             softcap=0.0, alibi_slopes=None, doc_ids=None, stream=None):
    """Attention backward.  q, o, dout [B,H,Sq,D] bf16, k/v [B,Hkv,Sk,D] bf16, lse fp32
    [B,H,Sq] from the forward.  Returns (dq [B,H,Sq,D], dk [B,Hkv,Sk,D], dv [B,Hkv,Sk,D])."""
    lib = load()
    B, H, Hkv, Sq, Sk, D = _check_qkv(q, k, v, torch.bfloat16, gqa=True)
    _check_mods(q, H, B, Sk, alibi_slopes, doc_ids)
    _need(o, "o", torch.bfloat16, (B, H, Sq, D), q.device)
    _need(dout, "dout", torch.bfloat16, (B, H, Sq, D), q.device)
    _need(lse, "lse", torch.float32, (B, H, Sq), q.device)
    outs = []
    for name, t, shape in (("dq", dq, (B, H, Sq, D)), ("dk", dk, (B, Hkv, Sk, D)), ("dv", dv, (B, Hkv, Sk, D))):
        if t is None:
            t = torch.empty(shape, dtype=torch.bfloat16, device=q.device)
        else:
            _need(t, name, torch.bfloat16, shape, q.device)
        outs.append(t)
    dq, dk, dv = outs
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                      B, H, Hkv, Sq, Sk, D, float(scale), int(mask_kind), int(window), float(softcap),
                      _ptr(alibi_slopes), _ptr(doc_ids), _stream(stream))
    check(rc, "attn_bwd")
    return dq, dk, dv


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, o=None, lse=None,
                    scale=None, mask_kind=MASK_NONE, window=0, softcap=0.0, alibi_slopes=None, stream=None):
    """Packed variable-length sequences.  q [Tq,H,D], k/v [Tk,Hkv,D] bf16; cu_seqlens_* int32
    [nseq+1] on the same device.  Returns (o bf16 [Tq,H,D], lse fp32 [H,Tq])."""
    lib = load()
    for name, t in (("q", q), ("k", k)):
        if not isinstance(t, torch.Tensor) or t.dim() != 3 or t.device.type != "cuda":
            raise ValueError(f"{name}: expected a 3-d CUDA tensor [T, heads, D]")
    Tq, H, D = q.shape
    Tk, Hkv = k.shape[0], k.shape[1]
    if Hkv < 1 or H % Hkv != 0:
        raise ValueError(f"k: {Hkv} key/value heads do not divide {H} query heads")
    _need(q, "q", torch.bfloat16, (Tq, H, D), q.device)
    _need(k, "k", torch.bfloat16, (Tk, Hkv, D), q.device)
    _need(v, "v", torch.bfloat16, (Tk, Hkv, D), q.device)
    if not isinstance(cu_seqlens_q, torch.Tensor) or cu_seqlens_q.dim() != 1:
        raise ValueError("cu_seqlens_q: expected a 1-d int32 tensor [nseq + 1]")
    nseq = cu_seqlens_q.shape[0] - 1
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, (nseq + 1,), q.device)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, (nseq + 1,), q.device)
    _check_mods(q, H, 1, Tk, alibi_slopes, None)
    if o is None:
        o = torch.empty(Tq, H, D, dtype=torch.bfloat16, device=q.device)
    else:
        _need(o, "o", torch.bfloat16, (Tq, H, D), q.device)
    if lse is None:
        lse = torch.empty(H, Tq, dtype=torch.float32, device=q.device)
    else:
        _need(lse, "lse", torch.float32, (H, Tq), q.device)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = lib.attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q),
                             _ptr(cu_seqlens_k), nseq, int(max_seqlen_q), int(max_seqlen_k), Tq, Tk, H, Hkv, D,
                             float(scale), int(mask_kind), int(window), float(softcap), _ptr(alibi_slopes),
                             _stream(stream))
    check(rc, "attn_fwd_varlen")
    return o, lse


def attn_fwd_noalloc(q, k, v, o, lse, scale=None, mask_kind=MASK_NONE, window=0, softcap=0.0,
                     alibi_slopes=None, doc_ids=None, stream=None):
    """attn_fwd without any device allocation inside the call: the caller passes the
    outputs, and the document-mask tile map uses the library's fixed per-device array
    (see include/attn.h).  For callers that cannot allocate during the call."""
    lib = load()
    B, H, Sq, Sk, D = _check_qkv(q, k, v, torch.bfloat16)
    _check_mods(q, H, B, Sk, alibi_slopes, doc_ids)
    if o is None or lse is None:
        raise ValueError("attn_fwd_noalloc: the caller passes o and lse (nothing is allocated)")
    _out(q, o, lse)
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
    if doc_ids is not None:
        _need(doc_ids, "doc_ids", torch.int32, (B, Sk), torch.device(device))
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
    B, H, Sq, Sk, D = _check_qkv(q, k, v, torch.bfloat16)
    _check_mods(q, H, B, Sk, alibi_slopes, doc_ids)
    cs, es = tile_map_shape(B, Sq, Sk)
    _need(counts, "counts", torch.int32, cs, q.device)
    _need(entries, "entries", torch.int32, es, q.device)
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
    if not isinstance(x, torch.Tensor) or x.dim() != 4 or x.device.type != "cuda":
        raise ValueError("x: expected a 4-d CUDA tensor [B, H, S, D]")
    B, H, S, D = x.shape
    _need(x, "x", torch.float32, (B, H, S, D), x.device)
    if xq is None:
        xq = torch.empty(B, H, S, D, dtype=torch.uint8, device=x.device)
    else:
        _need(xq, "xq", torch.uint8, (B, H, S, D), x.device)
    if scales is None:
        scales = torch.empty(B, H, (S + 127) // 128, dtype=torch.float32, device=x.device)
    else:
        _need(scales, "scales", torch.float32, (B, H, (S + 127) // 128), x.device)
    rc = lib.attn_quantize_e4m3(_ptr(x), _ptr(xq), _ptr(scales), B, H, S, D, _stream(stream))
    check(rc, "attn_quantize_e4m3")
    return xq, scales


def attn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o=None, lse=None, scale=None,
                 mask_kind=MASK_NONE, window=0, softcap=0.0, alibi_slopes=None, doc_ids=None,
                 stream=None):
    lib = load()
    B, H, Sq, Sk, D = _check_qkv(q8, k8, v8, torch.uint8)
    _check_mods(q8, H, B, Sk, alibi_slopes, doc_ids)
    _need(q_scale, "q_scale", torch.float32, (B, H, (Sq + 127) // 128), q8.device)
    _need(k_scale, "k_scale", torch.float32, (B, H, (Sk + 127) // 128), q8.device)
    _need(v_scale, "v_scale", torch.float32, (B, H, (Sk + 127) // 128), q8.device)
    o, lse = _out(q8, o, lse)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = lib.attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
                          _ptr(o), _ptr(lse), B, H, Sq, Sk, D, float(scale), int(mask_kind), int(window),
                          float(softcap), _ptr(alibi_slopes), _ptr(doc_ids), _stream(stream))
    check(rc, "attn_fwd_fp8")
    return o, lse


def mxfp4_shapes(B, H, S, transpose=False):
    """Shapes of (codes, scale atoms) that attn_quantize_mxfp4 writes for a [B,H,S,128] input."""
    nt = (S + 127) // 128
    if transpose:
        return (B, H, 128, nt * 64), (B, H, nt, 512)
    return (B, H, S, 64), (B, H, nt, 512)


def attn_quantize_mxfp4(x, transpose=False, xq=None, x_sf=None, stream=None):
    """bf16 [B,H,S,128] -> (e2m1 codes uint8, E8M0 scale atoms uint8), MXFP4 (32-element
    blocks).  transpose=True stores the codes as rows of D holding the keys (the layout V
    takes in attn_fwd_fp4)."""
    lib = load()
    if not isinstance(x, torch.Tensor) or x.dim() != 4 or x.device.type != "cuda":
        raise ValueError("x: expected a 4-d CUDA tensor [B, H, S, 128]")
    B, H, S, D = x.shape
    if D != 128:
        raise ValueError("attn_quantize_mxfp4 needs D = 128")
    _need(x, "x", torch.bfloat16, (B, H, S, D), x.device)
    qshape, sshape = mxfp4_shapes(B, H, S, transpose)
    if xq is None:
        xq = torch.empty(qshape, dtype=torch.uint8, device=x.device)
    else:
        _need(xq, "xq", torch.uint8, qshape, x.device)
    if x_sf is None:
        x_sf = torch.empty(sshape, dtype=torch.uint8, device=x.device)
    else:
        _need(x_sf, "x_sf", torch.uint8, sshape, x.device)
    rc = lib.attn_quantize_mxfp4(_ptr(x), _ptr(xq), _ptr(x_sf), B, H, S, D, 1 if transpose else 0, _stream(stream))
    check(rc, "attn_quantize_mxfp4")
    return xq, x_sf


def attn_fwd_fp4(q4, q_sf, k4, k_sf, vt4, v_sf, Sk, o=None, lse=None, scale=None, stream=None):
    """FP4 forward with Direct-P (no mask) on attn_quantize_mxfp4 outputs: q4/q_sf from Q,
    k4/k_sf from K, vt4/v_sf from V with transpose=True; Sk is the key count.  Grouped heads
    when K/V have fewer heads than Q.  Returns (o bf16 [B,H,Sq,128], lse fp32 [B,H,Sq])."""
    lib = load()
    for name, t in (("q4", q4), ("k4", k4), ("vt4", vt4)):
        if not isinstance(t, torch.Tensor) or t.dim() != 4 or t.device.type != "cuda":
            raise ValueError(f"{name}: expected a 4-d CUDA tensor")
    B, H, Sq, _ = q4.shape
    Hkv = k4.shape[1]
    if Hkv <= 0 or H % Hkv != 0:
        raise ValueError("the query heads must be a multiple of the key/value heads")
    qs, qsf = mxfp4_shapes(B, H, Sq)
    ks, ksf = mxfp4_shapes(B, Hkv, Sk)
    vs, vsf = mxfp4_shapes(B, Hkv, Sk, transpose=True)
    _need(q4, "q4", torch.uint8, qs, q4.device)
    _need(q_sf, "q_sf", torch.uint8, qsf, q4.device)
    _need(k4, "k4", torch.uint8, ks, q4.device)
    _need(k_sf, "k_sf", torch.uint8, ksf, q4.device)
    _need(vt4, "vt4", torch.uint8, vs, q4.device)
    _need(v_sf, "v_sf", torch.uint8, vsf, q4.device)
    if o is None:
        o = torch.empty(B, H, Sq, 128, dtype=torch.bfloat16, device=q4.device)
    else:
        _need(o, "o", torch.bfloat16, (B, H, Sq, 128), q4.device)
    if lse is None:
        lse = torch.empty(B, H, Sq, dtype=torch.float32, device=q4.device)
    else:
        _need(lse, "lse", torch.float32, (B, H, Sq), q4.device)
    scale = 1.0 / math.sqrt(128) if scale is None else scale
    rc = lib.attn_fwd_fp4(_ptr(q4), _ptr(k4), _ptr(vt4), _ptr(q_sf), _ptr(k_sf), _ptr(v_sf), _ptr(o), _ptr(lse),
                          B, H, Hkv, Sq, Sk, float(scale), _stream(stream))
    check(rc, "attn_fwd_fp4")
    return o, lse


def attn_get_status(stream=None) -> int:
    return load().attn_get_status(_stream(stream))


def attn_shutdown() -> None:
    load().attn_shutdown()

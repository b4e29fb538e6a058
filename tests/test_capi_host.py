"""Host-side checks of the C-ABI that need no GPU: the library loads, exports every symbol
include/attn.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from tiled_attention_14_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "attn.h")).read()
    return re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", src)


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = _declared()
    assert set(names) == set(_lib.SIGNATURES), (names, sorted(_lib.SIGNATURES))
    for n in names:
        assert getattr(lib, n) is not None


def test_strerror_is_static_text():
    for code in (0, -1, -2, -3, -4, -5, 99):
        assert isinstance(_lib.strerror(code), str) and _lib.strerror(code)


A = 4096  # a fake, 16-byte aligned "device" address: argument checks fail before any use


def _fwd(**kw):
    args = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=1, Sq=128, Sk=128, D=128, scale=0.1, mask=0,
                window=0, softcap=0.0, alibi=None, doc=None)
    args.update(kw)
    lib = _lib.load()
    return lib.attn_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["H"],
                        args["Sq"], args["Sk"], args["D"], args["scale"], args["mask"], args["window"],
                        args["softcap"], args["alibi"], args["doc"], None)


@pytest.mark.parametrize("kw", [
    dict(q=None), dict(o=None), dict(lse=None), dict(k=A + 8), dict(D=96), dict(D=256), dict(Sq=0),
    dict(Sk=-1), dict(B=0), dict(H=0), dict(scale=float("nan")), dict(scale=0.0), dict(scale=-1.0),
    dict(scale=float("inf")), dict(mask=8), dict(mask=2, window=0), dict(mask=4),
    dict(mask=4, doc=A, Sk=256), dict(softcap=float("inf")), dict(Sq=(1 << 20) + 1),
    dict(alibi=A + 4), dict(doc=A + 4, mask=4)])
def test_bad_arguments_rejected(kw):
    assert _fwd(**kw) == _lib.ATTN_ERR_INVALID


def test_bad_arguments_other_entry_points():
    lib = _lib.load()
    # the pair kernel takes BF16 with D = 128 only
    assert lib.attn_fwd_pair(A, A, A, A, A, 1, 1, 1, 128, 128, 64, 0.1, 0, 0, 0.0, None, None, None) == \
        _lib.ATTN_ERR_INVALID
    assert lib.attn_fwd_pair(A, A, A, A, A, 1, 2, 3, 128, 128, 128, 0.1, 0, 0, 0.0, None, None, None) == \
        _lib.ATTN_ERR_INVALID
    assert lib.attn_quantize_e4m3(A, A, A, 1, 1, 128, 96 + 8, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_quantize_e4m3(None, A, A, 1, 1, 128, 64, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_tile_map_build(None, A, 1, 128, 128, 0, 0, None, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_tile_map_build(A, A, 1, 128, 256, 4, 0, A, None) == _lib.ATTN_ERR_INVALID
    args = [A, A, A, A, A, 1, 1, 128, 128, 128, 0.1, 0, 0, 0.0, None, None]
    assert lib.attn_fwd_with_map(*args, None, A, None) == _lib.ATTN_ERR_INVALID
    fp8 = [A, A, A, A, A, A, A, A, 1, 1, 128, 128, 64, 0.1, 0, 0, 0.0, None, None, None]
    assert lib.attn_fwd_fp8(*fp8) == _lib.ATTN_ERR_INVALID          # D = 64 unsupported for FP8
    fp8[3] = None
    fp8[12] = 128
    assert lib.attn_fwd_fp8(*fp8) == _lib.ATTN_ERR_INVALID          # missing scales


@pytest.mark.parametrize("i,val", [(0, None), (3, None), (5, None), (6, None), (7, None), (2, A + 8),
                                   (8, 0), (9, 0), (10, 3), (11, 0), (12, -1), (11, (1 << 20) + 1),
                                   (13, 0.0), (13, float("nan"))])
def test_fp4_forward_rejects_bad_arguments(i, val):
    # q4, k4, vt4, q_sf, k_sf, v_sf, o, lse, B, H, H_kv, Sq, Sk, scale
    args = [A, A, A, A, A, A, A, A, 1, 2, 1, 128, 128, 0.1]
    args[i] = val
    assert _lib.load().attn_fwd_fp4(*args, None) == _lib.ATTN_ERR_INVALID


@pytest.mark.parametrize("kw", [dict(x=None), dict(D=64), dict(S=0), dict(transpose=2), dict(xq=A + 4),
                                dict(S=(1 << 20) + 1)])
def test_mxfp4_quantiser_rejects_bad_arguments(kw):
    a = dict(x=A, xq=A, sf=A, B=1, H=1, S=128, D=128, transpose=0)
    a.update(kw)
    assert _lib.load().attn_quantize_mxfp4(a["x"], a["xq"], a["sf"], a["B"], a["H"], a["S"], a["D"],
                                           a["transpose"], None) == _lib.ATTN_ERR_INVALID


def test_wrapper_raises_on_missing_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError):
        _lib.load()


def test_tmem_moves_header_is_generated():
    """csrc/tmem_moves.cuh is what tiled_attention_14_b200/gen_tmem_moves.py writes."""
    from tiled_attention_14_b200 import gen_tmem_moves
    assert gen_tmem_moves.main(["--check"]) == 0


def test_binding_rejects_host_tensors_and_bad_outputs():
    """The binding checks tensors before it passes bare pointers to the library."""
    import torch
    import tiled_attention_14_b200 as ta
    q = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ta.attn_fwd(q, q, q)                         # host tensors: there is no CPU path
    with pytest.raises(ValueError):
        ta.attn_fwd_noalloc(q, q, q, None, None)
    meta = torch.empty(1, 1, 128, 128, dtype=torch.bfloat16, device="meta")
    with pytest.raises(ValueError):
        ta.attn_fwd(meta, meta, meta)
    with pytest.raises(ValueError):
        ta.attn_quantize_e4m3(torch.zeros(1, 1, 128, 128))
    with pytest.raises(ValueError):
        ta.attn_quantize_mxfp4(q)                    # host tensor
    u8 = torch.zeros(1, 1, 128, 64, dtype=torch.uint8)
    with pytest.raises(ValueError):
        ta.attn_fwd_fp4(u8, u8, u8, u8, u8, u8, 128)    # host tensors


def test_mxfp4_shapes():
    """Storage shapes of the MXFP4 tensors: 64 bytes per row of 128 elements; V transposed with
    its keys padded to 128; one 512-byte scale atom per 128 rows (or keys)."""
    import tiled_attention_14_b200 as ta
    assert ta.mxfp4_shapes(2, 3, 300) == ((2, 3, 300, 64), (2, 3, 3, 512))
    assert ta.mxfp4_shapes(2, 3, 300, transpose=True) == ((2, 3, 128, 192), (2, 3, 3, 512))
    assert ta.mxfp4_shapes(1, 1, 1, transpose=True) == ((1, 1, 128, 64), (1, 1, 1, 512))


ABL_SIGNATURES = {
    "attn_ablation_set": (ctypes.c_int, [ctypes.c_float]),
    "attn_ablation_counts": (ctypes.c_int, [ctypes.c_void_p]),
    "attn_ablation_sw_exp_every": (ctypes.c_int, []),
}


def test_ablation_builds_export_their_header():
    """The ablation builds export attn.h's symbols and include/attn_ablation.h's; the product
    build exports none of the latter."""
    from tiled_attention_14_b200 import build
    src = open(os.path.join(ROOT, "include", "attn_ablation.h")).read()
    names = set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", src))
    assert names == set(ABL_SIGNATURES)
    for so in build.ABLATIONS:
        lib = _lib.open_library(os.path.join(os.path.dirname(_lib.LIB_PATH), so))
        for n in names:
            assert getattr(lib, n) is not None
        fn = lib.attn_ablation_sw_exp_every
        fn.restype = ctypes.c_int
        assert fn() == (4 if "sw4" in so else 0)
        set_tau = lib.attn_ablation_set
        set_tau.restype, set_tau.argtypes = ABL_SIGNATURES["attn_ablation_set"]
        assert set_tau(9.0) == _lib.ATTN_ERR_INVALID and set_tau(-1.0) == _lib.ATTN_ERR_INVALID
    product = _lib.load()
    for n in names:
        with pytest.raises(AttributeError):
            getattr(product, n)

"""attn_fwd_noalloc: the entry point for callers that cannot allocate device memory during
a call (a framework whose caching allocator owns device memory, a serving loop where an
allocation could synchronise the device, a fixed memory budget).  Its document-mask tile
map lives in a fixed per-device array instead of a per-call workspace.

The GPU test checks its output against attn_fwd's on the same inputs, on two calls in a
row (the second call finds the array holding the first call's map).  Both entry points run
the same kernel on the same tile map, so the outputs must be equal bit for bit; a
tolerance could hide a stale map.  It also checks, through the device's default memory
pool (where attn_fwd's stream-ordered workspace comes from), that the two calls allocate
nothing.  This file is named to be collected last."""
import math

import numpy as np
import pytest
import torch

from attn_workloads import MASK_CAUSAL, MASK_DOC, MASK_NONE, doc_ids_from_lengths, make_doc_ids, make_qkv
from tiled_attention_14_b200 import _lib

A = 4096   # fake 16-byte aligned address: the size check fails before any device use


def test_rejects_maps_larger_than_the_fixed_array():
    lib = _lib.load()
    # B=64, S=2^20 needs a 64*4096*8192*4-byte map: far above the 4 MiB array
    rc = lib.attn_fwd_noalloc(A, A, A, A, A, 64, 1, 1 << 20, 1 << 20, 128, 0.1, MASK_DOC, 0, 0.0, None, A, None)
    assert rc == _lib.ATTN_ERR_INVALID


def test_rejects_document_batches_beyond_the_grid_limit():
    lib = _lib.load()
    rc = lib.attn_fwd_noalloc(A, A, A, A, A, 65536, 1, 128, 128, 128, 0.1, MASK_DOC, 0, 0.0, None, A, None)
    assert rc == _lib.ATTN_ERR_INVALID
    rc = lib.attn_fwd(A, A, A, A, A, 65536, 1, 128, 128, 128, 0.1, MASK_DOC, 0, 0.0, None, A, None)
    assert rc == _lib.ATTN_ERR_INVALID


def _pool_high_water(reset: bool) -> int:
    """Bytes high-water mark of the current device's default memory pool (cudaMallocAsync
    draws from it); optionally reset it to the current use first."""
    from cuda.bindings import runtime as rt
    err, dev = rt.cudaGetDevice()
    assert err == rt.cudaError_t.cudaSuccess
    err, pool = rt.cudaDeviceGetDefaultMemPool(dev)
    assert err == rt.cudaError_t.cudaSuccess
    attr = rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh
    if reset:
        from cuda.bindings import driver as drv
        (err,) = rt.cudaMemPoolSetAttribute(pool, attr, drv.cuuint64_t(0))
        assert err == rt.cudaError_t.cudaSuccess
    err, val = rt.cudaMemPoolGetAttribute(pool, attr)
    assert err == rt.cudaError_t.cudaSuccess
    return int(val)


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["doc_bench_rows", "doc_ragged_causal", "plain_causal"])
def test_noalloc_matches_attn_fwd_twice(case):
    import tiled_attention_14_b200 as ta
    if case == "doc_bench_rows":
        B, H, S, D, mask = 2, 4, 8192, 128, MASK_DOC
        doc = make_doc_ids(B, S)
    elif case == "doc_ragged_causal":
        lens = [300, 129, 1, 450, 144]
        B, H, S, D, mask = 2, 2, sum(lens), 64, MASK_DOC | MASK_CAUSAL
        doc = torch.from_numpy(np.stack([doc_ids_from_lengths(lens), doc_ids_from_lengths(lens[::-1])]))
    else:
        B, H, S, D, mask = 1, 2, 1000, 128, MASK_CAUSAL
        doc = None
    q, k, v = (t.cuda() for t in make_qkv(B, H, S, S, D, seed=31))
    docd = None if doc is None else doc.cuda().contiguous()
    ref_o, ref_l = ta.attn_fwd(q, k, v, mask_kind=mask, doc_ids=docd)
    outs = [(torch.empty_like(ref_o), torch.empty_like(ref_l)) for _ in range(2)]
    # one warm-up call: the first call on a device may load the library's device code
    ta.attn_fwd_noalloc(q, k, v, *outs[0], mask_kind=mask, doc_ids=docd)
    torch.cuda.synchronize()
    for o, lse in outs:
        o.fill_(7.0)
        lse.fill_(7.0)
    torch.cuda.synchronize()
    _pool_high_water(reset=True)
    for o, lse in outs:
        ta.attn_fwd_noalloc(q, k, v, o, lse, mask_kind=mask, doc_ids=docd)
        torch.cuda.synchronize()
        assert ta.attn_get_status() == 0
    assert _pool_high_water(reset=False) == 0, "attn_fwd_noalloc drew memory from the default pool"
    for o, lse in outs:
        assert torch.equal(o, ref_o)
        assert torch.equal(lse, ref_l)

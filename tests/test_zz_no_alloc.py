"""attn_fwd_noalloc: the entry point for callers that cannot allocate device memory during
a call (a framework whose caching allocator owns device memory, a serving loop where an
allocation could synchronise the device, a fixed memory budget).  Its document-mask tile
map lives in a fixed per-device array instead of a per-call workspace.

The GPU test checks its output against attn_fwd's on the same inputs, on two calls in a
row (the second call finds the array holding the first call's map), with the tolerance the
parity tests use.  This file is named to be collected last."""
import math

import numpy as np
import pytest
import torch

from attn_workloads import MASK_CAUSAL, MASK_DOC, MASK_NONE, doc_ids_from_lengths, make_doc_ids, make_qkv
from tests.gpu_helpers import TOL_LSE_BF16, TOL_O_BF16
from tiled_attention_14_b200 import _lib

A = 4096   # fake 16-byte aligned address: the size check fails before any device use


def test_rejects_maps_larger_than_the_fixed_array():
    lib = _lib.load()
    # B=64, S=2^20 needs a 64*4096*8192*4-byte map: far above the 4 MiB array
    rc = lib.attn_fwd_noalloc(A, A, A, A, A, 64, 1, 1 << 20, 1 << 20, 128, 0.1, MASK_DOC, 0, 0.0, None, A, None)
    assert rc == _lib.ATTN_ERR_INVALID


def _compare(o1, l1, o2, l2):
    d_o = (o1.float() - o2.float()).abs().max().item()
    fin = torch.isfinite(l1)
    assert torch.equal(fin, torch.isfinite(l2))
    d_l = (l1[fin] - l2[fin]).abs().max().item() if fin.any() else 0.0
    assert d_o <= TOL_O_BF16 and d_l <= TOL_LSE_BF16, (d_o, d_l)


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
    for _ in range(2):
        o = torch.empty_like(ref_o)
        lse = torch.empty_like(ref_l)
        ta.attn_fwd_noalloc(q, k, v, o, lse, mask_kind=mask, doc_ids=docd)
        torch.cuda.synchronize()
        assert ta.attn_get_status() == 0
        _compare(o, lse, ref_o, ref_l)

"""GPU tile-map builder and e4m3 quantiser: bit-exact against the oracle."""
import numpy as np
import pytest
import torch

from attn_workloads import (MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, doc_ids_from_lengths,
                            make_doc_ids, make_fp8_source)
from oracle import e4m3
from oracle.tile_map import tile_map

pytestmark = pytest.mark.gpu


def _check_map(B, Sq, Sk, mask, window, doc):
    import tiled_attention_14_b200 as ta
    docd = None if doc is None else doc.cuda()
    counts, entries = ta.attn_tile_map_build(B, Sq, Sk, mask, window, docd)
    torch.cuda.synchronize()
    c_ref, e_ref = tile_map(B, Sq, Sk, mask, window, doc)
    c = counts.cpu().numpy()
    e = entries.cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(c, c_ref)
    for b in range(B):
        for qb in range(c.shape[1]):
            n = c[b, qb]
            np.testing.assert_array_equal(e[b, qb, :n], e_ref[b, qb, :n])


@pytest.mark.parametrize("Sq,Sk,mask,window", [
    (1024, 1024, MASK_CAUSAL, 0), (700, 700, MASK_CAUSAL | MASK_WINDOW, 200), (700, 900, MASK_WINDOW, 130),
    (300, 300, MASK_NONE, 0), (333, 901, MASK_CAUSAL, 0), (901, 333, MASK_CAUSAL | MASK_WINDOW, 1)])
def test_tile_map_positional(Sq, Sk, mask, window):
    _check_map(2, Sq, Sk, mask, window, None)


@pytest.mark.parametrize("mask", [MASK_DOC, MASK_DOC | MASK_CAUSAL, MASK_DOC | MASK_CAUSAL | MASK_WINDOW])
def test_tile_map_documents(mask):
    lens = [[300, 129, 1, 450, 144, 2000], [1024, 1000, 1, 1, 998]]
    S = sum(lens[0])
    doc = torch.from_numpy(np.stack([doc_ids_from_lengths(l) for l in lens]))
    _check_map(2, S, S, mask, 300, doc)


def test_tile_map_documents_unsorted():
    rng = np.random.default_rng(0)
    doc = torch.from_numpy(rng.integers(0, 4, size=(2, 777)).astype(np.int32))
    _check_map(2, 777, 777, MASK_DOC, 0, doc)
    # long runs with a repeated id
    d = np.concatenate([np.zeros(300), np.ones(200), np.zeros(277)]).astype(np.int32)
    _check_map(1, 777, 777, MASK_DOC | MASK_CAUSAL, 0, torch.from_numpy(d[None]))


def test_tile_map_benchmark_documents():
    doc = make_doc_ids(2, 8192)
    _check_map(2, 8192, 8192, MASK_DOC, 0, doc)


@pytest.mark.parametrize("B,H,S,D", [(2, 3, 300, 128), (1, 2, 128, 64), (1, 1, 1000, 16)])
def test_quantiser_bit_exact(B, H, S, D):
    import tiled_attention_14_b200 as ta
    g = torch.Generator().manual_seed(S)
    x = torch.randn(B, H, S, D, generator=g) * 3
    x[0, 0, :128] = 0.0                       # a zero block
    x[-1, -1, -1, 0] = 1e5                    # an outlier
    xq, sc = ta.attn_quantize_e4m3(x.cuda())
    torch.cuda.synchronize()
    codes, scales = e4m3.quantize_blocks(x)
    np.testing.assert_array_equal(xq.cpu().numpy(), codes)
    np.testing.assert_array_equal(sc.cpu().numpy(), scales)


def test_quantiser_benchmark_inputs():
    import tiled_attention_14_b200 as ta
    q, _, _ = make_fp8_source(1, 16, 2048, 128, seed=0)
    xq, sc = ta.attn_quantize_e4m3(q.cuda())
    torch.cuda.synchronize()
    codes, scales = e4m3.quantize_blocks(q)
    np.testing.assert_array_equal(xq.cpu().numpy(), codes)
    np.testing.assert_array_equal(sc.cpu().numpy(), scales)

"""The small parity cases under the bounds-checked debug build (libattn_debug.so): every
TMA copy and TMEM move of the forward, FP8, packed-sequence and backward kernels is checked
before it is issued (shared-memory range and alignment, coordinate alignment, TMEM columns
and lane quarter).  A failed check would show as ATTN_ERR_CHECK from attn_get_status; the
helpers assert a zero status after every call, and every case still matches the oracle."""
import os

import numpy as np
import pytest
import torch

from attn_workloads import MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, doc_ids_from_lengths
from tiled_attention_14_b200 import _lib
from tiled_attention_14_b200.build import DEBUG

pytestmark = pytest.mark.gpu


@pytest.fixture
def debug_library(monkeypatch):
    lib = _lib.open_library(os.path.join(os.path.dirname(_lib.LIB_PATH), next(iter(DEBUG))))
    monkeypatch.setattr(_lib, "_lib", lib)
    yield lib


def test_forward_cases(debug_library):
    from tests import test_gpu_parity as t
    t._run(1, 3, 300, 300, 64, seed=1)
    t._run(2, 2, 520, 200, 128, MASK_CAUSAL, seed=2)
    t._run(1, 2, 700, 700, 128, MASK_WINDOW | MASK_CAUSAL, window=100, seed=3)
    t._run(1, 2, 520, 520, 128, MASK_NONE, softcap=50.0, seed=4)
    t._run(1, 4, 600, 600, 128, MASK_CAUSAL, alibi=True, seed=5)
    lens = [300, 129, 1, 450, 144]
    doc = torch.from_numpy(np.stack([doc_ids_from_lengths(lens), doc_ids_from_lengths(lens[::-1])]))
    t._run(2, 2, sum(lens), sum(lens), 128, MASK_DOC, doc=doc, seed=6)


def test_fp8_and_packed_and_grouped(debug_library):
    from tests import test_gpu_fp8 as f
    from tests import test_gpu_gqa_varlen as g
    f._fp8_case(1, 4, 300, 128, MASK_CAUSAL, seed=7)
    g._varlen_case([200, 0, 513, 77], [350, 40, 257, 77], 4, 2, 128, MASK_CAUSAL, seed=8)
    g.test_gqa(16, 4, MASK_CAUSAL, 64)


def test_backward_cases(debug_library):
    from tests import test_gpu_bwd as b
    b._run(1, 2, 2, 300, 300, 128, MASK_CAUSAL, seed=9)
    b._run(2, 4, 1, 260, 260, 64, MASK_NONE, softcap=20.0, alibi=True, seed=10)


def test_fp4_cases(debug_library):
    # the FP4 kernel's TMA boxes, bulk scale copies, scale-factor copies to tensor memory and
    # TMEM moves, and the MXFP4 quantisers, all checked
    from tests import test_gpu_fp4 as f
    from attn_workloads import make_qkv
    f._check(*make_qkv(1, 2, 300, 333, 128, seed=11))
    f._check(*make_qkv(1, 4, 256, 200, 128, seed=12, Hkv=2))

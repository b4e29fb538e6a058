"""Bounded waits: when a signal inside the kernel never comes, the kernel gives up after
its time limit, records ATTN_ERR_TIMEOUT in the device status word, frees its tensor
memory and returns — no trap, no hang — and the CUDA context stays usable.

The test hook makes the second softmax group of every CTA skip its first P-ready signal,
so the MMA issuer's wait for it runs out (limit 200 ms here)."""
import pytest
import torch

from attn_workloads import MASK_CAUSAL, make_qkv
from tests.gpu_helpers import compare, oracle_eav, to_dev

pytestmark = pytest.mark.gpu


def test_skipped_signal_times_out_and_context_survives():
    import tiled_attention_14_b200 as ta
    from tiled_attention_14_b200 import _lib
    lib = _lib.load()
    q, k, v = make_qkv(1, 2, 640, 640, 128, seed=41)
    qd, kd, vd = to_dev(q, k, v)
    assert ta.attn_get_status() == _lib.ATTN_OK
    lib.attn_debug_set_fault(1, 200)
    try:
        ta.attn_fwd(qd, kd, vd, mask_kind=MASK_CAUSAL)
        assert ta.attn_get_status() == _lib.ATTN_ERR_TIMEOUT
    finally:
        lib.attn_debug_set_fault(0, 1000)
    # the status word was cleared by the read, and the context still runs kernels correctly
    assert ta.attn_get_status() == _lib.ATTN_OK
    o, lse = ta.attn_fwd(qd, kd, vd, mask_kind=MASK_CAUSAL)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == _lib.ATTN_OK
    O, L, E = oracle_eav(q, k, v, 1.0 / 128 ** 0.5, MASK_CAUSAL)
    compare(o, lse, O, L, eav=E)


def test_pair_kernel_skipped_signal_times_out_and_context_survives():
    """The same hook in the pair kernel: the odd CTA's first softmax warp skips its first
    P-ready arrival on the even CTA's barrier; the MMA issuer's wait runs out, the other CTA's
    waits run out in turn, both CTAs still meet at their final cluster barrier and free the
    pair's tensor memory."""
    import tiled_attention_14_b200 as ta
    from tiled_attention_14_b200 import _lib
    lib = _lib.load()
    q, k, v = make_qkv(1, 2, 640, 640, 128, seed=42)
    qd, kd, vd = to_dev(q, k, v)
    assert ta.attn_get_status() == _lib.ATTN_OK
    lib.attn_debug_set_fault(1, 200)
    try:
        ta.attn_fwd_pair(qd, kd, vd, mask_kind=MASK_CAUSAL)
        assert ta.attn_get_status() == _lib.ATTN_ERR_TIMEOUT
    finally:
        lib.attn_debug_set_fault(0, 1000)
    assert ta.attn_get_status() == _lib.ATTN_OK
    o, lse = ta.attn_fwd_pair(qd, kd, vd, mask_kind=MASK_CAUSAL)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == _lib.ATTN_OK
    O, L, E = oracle_eav(q, k, v, 1.0 / 128 ** 0.5, MASK_CAUSAL)
    compare(o, lse, O, L, eav=E)


def test_fp4_kernel_skipped_signal_times_out_and_context_survives():
    """The same hook in the FP4 kernel: query group 1 skips its first P-ready arrival; the
    MMA issuer's wait runs out, every role unwinds, and the next call is correct."""
    import tiled_attention_14_b200 as ta
    from tiled_attention_14_b200 import _lib
    from tests.test_gpu_fp4 import _check, _quantise_all
    lib = _lib.load()
    q, k, v = make_qkv(1, 2, 512, 512, 128, seed=43)
    q4, qsf, k4, ksf, v4, vsf = _quantise_all(q, k, v)
    assert ta.attn_get_status() == _lib.ATTN_OK
    lib.attn_debug_set_fault(1, 200)
    try:
        ta.attn_fwd_fp4(q4, qsf, k4, ksf, v4, vsf, 512)
        assert ta.attn_get_status() == _lib.ATTN_ERR_TIMEOUT
    finally:
        lib.attn_debug_set_fault(0, 1000)
    assert ta.attn_get_status() == _lib.ATTN_OK
    _check(q, k, v)

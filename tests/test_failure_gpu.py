"""Failure detection on the GPU without a fault: a device wait that runs out
(the watchdog self-test switch) and a corrupt BlockMask each end in a status the
host reads (FA_ERR_TIMEOUT / FA_ERR_BAD_BLOCKMASK), the kernel exits, and the
next forward on the same context is correct again."""

import time

import pytest
import torch

import oracle
from helpers import assert_forward_close, gpu_score

pytestmark = pytest.mark.gpu


def _fa():
    import block_sparse_attention_48_b200 as fa
    return fa


def _inputs(D, seed, ql=300, H=2):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((1, H, ql, D), generator=g).to(torch.bfloat16)
    k = torch.randn((1, H, ql, D), generator=g).to(torch.bfloat16)
    v = torch.randn((1, H, ql, D), generator=g).to(torch.bfloat16)
    return q, k, v


def _forward(q, k, v, score=("none",), bm=None):
    fa = _fa()
    if bm is None:
        bm = fa.create_block_mask("and", [("causal",)], 1, 1, q.shape[2], k.shape[2])
    o, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, score_mod=gpu_score(score))
    return o, lse


def _check_recovered(D, score=("none",), seed=5):
    fa = _fa()
    q, k, v = _inputs(D, seed)
    o, lse = _forward(q, k, v, score)
    assert fa.device_status() == fa.FA_OK
    o_ref, lse_ref = oracle.forward(q, k, v, "and", [("causal",)], None, score=score)
    assert_forward_close(o, lse, o_ref, lse_ref, f"recovered_d{D}")


@pytest.mark.parametrize("D,score", [(64, ("none",)), (128, ("none",)), (64, "bias")],
                         ids=["d64", "d128", "d64_bias"])
def test_watchdog_timeout_is_reported_and_context_survives(D, score):
    fa = _fa()
    assert fa.device_status() == fa.FA_OK
    q, k, v = _inputs(D, 3)
    if score == "bias":
        g = torch.Generator().manual_seed(4)
        score = ("bias", torch.randn((1, 2, 300, 300), generator=g).to(torch.bfloat16))
    fa.set_watchdog_ms(50)
    fa.set_selftest_stall(True)
    try:
        t0 = time.monotonic()
        _forward(q, k, v, score)
        status = fa.device_status()
        elapsed = time.monotonic() - t0
    finally:
        fa.set_selftest_stall(False)
        fa.set_watchdog_ms(0)
    assert status == fa.FA_ERR_TIMEOUT
    assert elapsed < 10.0
    # the status was cleared by the read, and the context still computes correctly
    assert fa.device_status() == fa.FA_OK
    _check_recovered(D, score)


def test_corrupt_block_mask_is_reported_without_fault():
    """Counts above nkv and negative / out-of-range kv indices are clamped in the
    kernel (no out-of-bounds read) and reported as FA_ERR_BAD_BLOCKMASK."""
    fa = _fa()
    q, k, v = _inputs(64, 7, ql=700)
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, 700, 700)
    nkv = bm.shape[3]
    bm.kv_num_blocks[0, 0, 0] = nkv + 5
    bm.kv_indices[0, 0, 1, 0] = -3
    bm.full_kv_indices[0, 0, 4, 0] = nkv + 100
    bm.full_kv_num_blocks[0, 0, 3] = -1
    _forward(q, k, v, bm=bm)
    assert fa.device_status() == fa.FA_ERR_BAD_BLOCKMASK
    assert fa.device_status() == fa.FA_OK
    _check_recovered(64)

"""The C ABI without a GPU: the library loads, exports every function that
include/flexattn.h declares, and rejects bad arguments before any CUDA call."""

import ctypes
import os
import re

import pytest

import block_sparse_attention_48_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flexattn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(fa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(fa.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fa.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings():
    assert fa.status_string(0) == "FA_OK"
    assert fa.status_string(fa.FA_ERR_TIMEOUT) == "FA_ERR_TIMEOUT"
    assert fa.status_string(fa.FA_ERR_BAD_BLOCKMASK) == "FA_ERR_BAD_BLOCKMASK"
    assert fa.status_string(99) == "FA_ERR_UNKNOWN"


def test_block_mask_shape():
    lib = fa.library()
    nq, nkv = ctypes.c_int32(), ctypes.c_int32()
    assert lib.fa_block_mask_shape(300, 513, 128, ctypes.byref(nq), ctypes.byref(nkv)) == 0
    assert (nq.value, nkv.value) == (3, 5)
    assert lib.fa_block_mask_shape(0, 0, 128, ctypes.byref(nq), ctypes.byref(nkv)) == 0
    assert (nq.value, nkv.value) == (0, 0)
    assert lib.fa_block_mask_shape(256, 256, 64, ctypes.byref(nq), ctypes.byref(nkv)) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_block_mask_shape(-1, 256, 128, ctypes.byref(nq), ctypes.byref(nkv)) == fa.FA_ERR_INVALID_ARG


def test_workspace_size():
    assert fa.library().fa_workspace_size() >= 4


def _bm(B=1, H=1, nq=2, nkv=2):
    d = fa.BlockMaskDesc()
    d.kv_num_blocks = d.kv_indices = d.full_kv_num_blocks = d.full_kv_indices = 4096
    d.B, d.H, d.nq, d.nkv, d.block_size, d.has_full = B, H, nq, nkv, 128, 1
    d.q_len = d.kv_len = 128 * nq
    return d


def test_create_block_mask_rejects_bad_arguments():
    lib = fa.library()
    m = fa.mask_desc("and", [("causal",)])
    d = _bm()
    call = lambda m_, B, H, ql, kl, bs: lib.fa_create_block_mask(ctypes.byref(m_) if m_ else None, B, H, ql, kl, bs,
                                                                  ctypes.byref(d), None)
    assert call(m, 0, 1, 256, 256, 128) == fa.FA_ERR_INVALID_ARG
    assert call(m, 1, 1, 256, 256, 64) == fa.FA_ERR_UNSUPPORTED
    assert call(None, 1, 1, 256, 256, 128) == fa.FA_ERR_INVALID_ARG
    bad = fa.mask_desc("and", [("causal",)])
    bad.kind[0] = 7
    assert call(bad, 1, 1, 256, 256, 128) == fa.FA_ERR_INVALID_ARG
    nodoc = fa.mask_desc("and", [("document",)])
    assert call(nodoc, 1, 1, 256, 256, 128) == fa.FA_ERR_INVALID_ARG
    bad_op = fa.mask_desc("and", [("causal",)])
    bad_op.op = 5
    assert call(bad_op, 1, 1, 256, 256, 128) == fa.FA_ERR_INVALID_ARG
    # batch and heads become grid extents: at most 65535 each
    assert call(m, 65536, 1, 256, 256, 128) == fa.FA_ERR_INVALID_ARG
    assert call(m, 1, 65536, 256, 256, 128) == fa.FA_ERR_INVALID_ARG


def _tensor(dims, data=4096):
    t = fa.TensorDesc()
    t.data = data
    st = [dims[1] * dims[2] * dims[3], dims[2] * dims[3], dims[3], 1]
    for i in range(4):
        t.dims[i], t.strides[i] = dims[i], st[i]
    return t


def _forward(q, k, v, o, bm, sm=None, ws=4096, ws_bytes=256):
    lib = fa.library()
    return lib.fa_forward(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.byref(bm),
                          ctypes.byref(sm) if sm is not None else None, ctypes.c_float(0.0), ctypes.byref(o),
                          None, ctypes.c_void_p(ws), ctypes.c_size_t(ws_bytes), None)


def test_forward_rejects_bad_arguments():
    q = _tensor([1, 2, 256, 64]); k = _tensor([1, 2, 256, 64]); v = _tensor([1, 2, 256, 64]); o = _tensor([1, 2, 256, 64])
    bm = _bm()
    # unsupported head dimension
    q32 = _tensor([1, 2, 256, 32]); k32 = _tensor([1, 2, 256, 32])
    assert _forward(q32, k32, k32, q32, bm) == fa.FA_ERR_UNSUPPORTED
    # GQA ratio
    assert _forward(_tensor([1, 3, 256, 64]), k, v, _tensor([1, 3, 256, 64]), bm) == fa.FA_ERR_INVALID_ARG
    # misaligned pointer and non-unit inner stride
    assert _forward(_tensor([1, 2, 256, 64], data=4098), k, v, o, bm) == fa.FA_ERR_INVALID_ARG
    qs = _tensor([1, 2, 256, 64]); qs.strides[3] = 2
    assert _forward(qs, k, v, o, bm) == fa.FA_ERR_INVALID_ARG
    # BlockMask built for another length, or with a batch extent that does not broadcast
    assert _forward(q, k, v, o, _bm(nq=3, nkv=3)) == fa.FA_ERR_INVALID_ARG
    assert _forward(q, k, v, o, _bm(B=3)) == fa.FA_ERR_INVALID_ARG
    # workspace too small / missing
    assert _forward(q, k, v, o, bm, ws_bytes=8) == fa.FA_ERR_INVALID_ARG
    assert _forward(q, k, v, o, bm, ws=0) == fa.FA_ERR_INVALID_ARG
    # score mods without their operands
    sm = fa.ScoreModDesc(); sm.kind = fa.SCORE["alibi"]
    assert _forward(q, k, v, o, bm, sm) == fa.FA_ERR_INVALID_ARG
    sm = fa.ScoreModDesc(); sm.kind = fa.SCORE["softcap"]; sm.softcap = 0.0
    assert _forward(q, k, v, o, bm, sm) == fa.FA_ERR_INVALID_ARG
    sm = fa.ScoreModDesc(); sm.kind = fa.SCORE["bias"]
    assert _forward(q, k, v, o, bm, sm) == fa.FA_ERR_INVALID_ARG
    sm = fa.ScoreModDesc(); sm.kind = 9
    assert _forward(q, k, v, o, bm, sm) == fa.FA_ERR_INVALID_ARG


def test_forward_rejects_expanded_dimensions():
    """A stride of 0 is accepted only on a size-1 dimension (an expanded tensor
    would make every head or batch read data other than the caller's); a bias may
    broadcast over batch and heads but not over queries."""
    q = _tensor([1, 2, 256, 64]); k = _tensor([1, 2, 256, 64]); v = _tensor([1, 2, 256, 64]); o = _tensor([1, 2, 256, 64])
    bm = _bm()
    for t in ("q", "k", "v", "o"):
        for dim in (0, 1, 2):
            ts = {n: _tensor([2, 2, 256, 64]) for n in "qkvo"}
            ts[t].strides[dim] = 0
            assert _forward(ts["q"], ts["k"], ts["v"], ts["o"], _bm(B=2)) == fa.FA_ERR_INVALID_ARG, (t, dim)
    sm = fa.ScoreModDesc(); sm.kind = fa.SCORE["bias"]; sm.bias = 4096
    for i, st in enumerate([2 * 256 * 256, 256 * 256, 0, 1]):
        sm.bias_strides[i] = st
    assert _forward(q, k, v, o, bm, sm) == fa.FA_ERR_INVALID_ARG


def test_backward_workspace_size_and_argument_checks():
    lib = fa.library()
    # status word + per 128-row query block its LSE and Delta rows (1 KB) + the fp32
    # dQ accumulator over the padded rows
    blocks = 2 * 3 * 1
    assert lib.fa_backward_workspace_size(2, 3, 100, 64) == 256 + blocks * 1024 + blocks * 128 * 64 * 4
    blocks = 1 * 2 * 3
    assert lib.fa_backward_workspace_size(1, 2, 257, 128) == 256 + blocks * 1024 + blocks * 128 * 128 * 4
    q = _tensor([1, 2, 256, 64]); k = _tensor([1, 2, 256, 64])
    bm = _bm()
    sm = fa.ScoreModDesc()
    ws = lib.fa_backward_workspace_size(1, 2, 256, 64)

    def call(ts, lse=4096, bm_=bm, ws_bytes=ws):
        return lib.fa_backward(*[ctypes.byref(t) for t in ts[:5]], ctypes.c_void_p(lse), ctypes.byref(bm_),
                               ctypes.byref(sm), ctypes.c_float(0.0), *[ctypes.byref(t) for t in ts[5:]],
                               ctypes.c_void_p(4096), ctypes.c_size_t(ws_bytes), None)
    base = [q, k, k, q, q, q, k, k]
    # the transposed view is missing (q_* pointers NULL)
    assert call(base) == fa.FA_ERR_INVALID_ARG
    bm_t = _bm()
    bm_t.q_num_blocks = bm_t.q_indices = bm_t.full_q_num_blocks = bm_t.full_q_indices = 4096
    # lse missing, workspace too small, dk of another shape, unsupported D
    assert call(base, bm_=bm_t, lse=0) == fa.FA_ERR_INVALID_ARG
    assert call(base, bm_=bm_t, ws_bytes=ws - 4) == fa.FA_ERR_INVALID_ARG
    assert call([q, k, k, q, q, q, _tensor([1, 2, 128, 64]), k], bm_=bm_t) == fa.FA_ERR_INVALID_ARG
    q32 = _tensor([1, 2, 256, 32])
    assert call([q32] * 8, bm_=bm_t) == fa.FA_ERR_UNSUPPORTED


def test_paged_and_decode_argument_checks():
    lib = fa.library()
    q = _tensor([1, 2, 256, 64]); o = _tensor([1, 2, 256, 64])
    pages = _tensor([6, 2, 128, 64])
    bm = _bm()
    sm = fa.ScoreModDesc()

    def paged(k, v, pt=4096, stride=2):
        return lib.fa_forward_paged(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.c_void_p(pt), stride,
                                    ctypes.byref(bm), ctypes.byref(sm), ctypes.c_float(0.0), ctypes.byref(o), None,
                                    ctypes.c_void_p(4096), ctypes.c_size_t(256), None)
    assert paged(pages, pages, pt=0) == fa.FA_ERR_INVALID_ARG           # no page table
    assert paged(pages, pages, stride=1) == fa.FA_ERR_INVALID_ARG       # shorter than nkv = 2
    bad = _tensor([6, 2, 64, 64])                                       # pages of 64 keys
    assert paged(bad, bad) == fa.FA_ERR_INVALID_ARG
    assert paged(pages, _tensor([5, 2, 128, 64])) == fa.FA_ERR_INVALID_ARG

    def decode(qq, k, oo, bm_, ws=1 << 20):
        return lib.fa_decode(ctypes.byref(qq), ctypes.byref(k), ctypes.byref(k), ctypes.byref(bm_), ctypes.byref(sm),
                             ctypes.c_float(0.0), ctypes.byref(oo), None, ctypes.c_void_p(4096), ctypes.c_size_t(ws),
                             None)
    q1 = _tensor([1, 32, 1, 64]); k1 = _tensor([1, 1, 256, 64])
    bm1 = _bm(nq=1, nkv=2)
    bm1.q_len, bm1.kv_len = 1, 256
    assert decode(q1, k1, q1, bm1) == fa.FA_ERR_UNSUPPORTED             # 32 query rows per kv head
    q4 = _tensor([1, 4, 1, 64])
    bmh = _bm(H=4, nq=1, nkv=2)
    bmh.q_len, bmh.kv_len = 1, 256
    assert decode(q4, k1, q4, bmh) == fa.FA_ERR_UNSUPPORTED             # per-head BlockMask
    assert lib.fa_decode_workspace_size(1, 4, 1, 1, 256, 64) >= 256


def test_empty_problem_enqueues_nothing():
    """q_len = 0: nothing to compute, returns FA_OK without touching the device."""
    q = _tensor([1, 2, 0, 64]); k = _tensor([1, 2, 256, 64]); o = _tensor([1, 2, 0, 64])
    bm = _bm(nq=0, nkv=2)
    bm.q_len, bm.kv_len = 0, 256
    assert _forward(q, k, k, o, bm) == fa.FA_OK


def test_watchdog_setting():
    assert fa.library().fa_set_watchdog_ms(-1) == fa.FA_ERR_INVALID_ARG
    fa.set_watchdog_ms(0)


def test_selftest_stall_setting():
    """The watchdog self-test switch is host state only: it can be set and cleared
    without a GPU."""
    assert fa.library().fa_set_selftest_stall(1) == fa.FA_OK
    fa.set_selftest_stall(False)

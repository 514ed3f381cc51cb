"""fa_backward on the GPU against the fp64 oracle's gradients, element by element.

Tolerance.  The pages state none for the backward pass; the forward's stated
O tolerance (2e-2 max-abs for O of magnitude ~1) is applied norm-wise to every
gradient: max |g - ref| <= 2e-2 * max |ref|.  The kernel rounds P and dS to bf16
(relative 2^-9) before the products dV = P^T dO, dK = dS^T Q and dQ = dS K, and
accumulates in fp32, so its error is a few 1e-3 of the largest gradient entry."""

import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from helpers import gpu_score

pytestmark = pytest.mark.gpu

G_REL = 2e-2


def _fa():
    import block_sparse_attention_48_b200 as fa
    return fa


def assert_grad_close(got, ref, what):
    g = got.float().cpu().numpy() if torch.is_tensor(got) else np.asarray(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite gradient"
    scale = np.abs(ref).max() if ref.size else 0.0
    err = np.abs(g - ref).max() if ref.size else 0.0
    assert err <= G_REL * max(scale, 1e-6), f"{what}: max|g-ref| = {err:.3e}, max|ref| = {scale:.3e}"
    return err / max(scale, 1e-30)


def _inputs(B, Hq, Hkv, ql, kl, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, ql, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, kl, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, kl, D), generator=g).to(torch.bfloat16)
    do = torch.randn((B, Hq, ql, D), generator=g).to(torch.bfloat16)
    return q, k, v, do


def _doc(B, L, seed):
    g = torch.Generator().manual_seed(seed)
    rows = []
    for b in range(B):
        lengths, acc = [], 0
        while acc < L:
            n = int(torch.randint(20, 400, (1,), generator=g))
            lengths.append(min(n, L - acc))
            acc += lengths[-1]
        rows.append(W.document_ids_from_lengths(lengths))
    return torch.stack(rows)


def _score(spec, B, Hq, ql, kl, seed):
    g = torch.Generator().manual_seed(seed + 7)
    if spec == "alibi":
        return ("alibi", W.alibi_slopes(Hq))
    if spec == "bias":
        return ("bias", torch.randn((B, Hq, ql, kl), generator=g).to(torch.bfloat16))
    if spec == "bias_softcap":
        return ("bias_softcap", (3 * torch.randn((B, Hq, ql, kl), generator=g)).to(torch.bfloat16), 4.0)
    return spec


def run_gpu(q, k, v, do, op, leaves, doc, score, bmB=1, split_full=True):
    fa = _fa()
    bm = fa.create_block_mask(op, leaves, bmB, 1, q.shape[2], k.shape[2], doc_ids=doc, transposed=True,
                              split_full=split_full)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    sm = gpu_score(score)
    o, lse = fa.flex_attention(qd, kd, vd, bm, score_mod=sm)
    dq, dk, dv = fa.flex_attention_backward(qd, kd, vd, o, lse, dod, bm, score_mod=sm)
    torch.cuda.synchronize()
    return dq, dk, dv


CASES = [
    # name, B, Hq, Hkv, q_len, kv_len, D, op, leaves, doc, score
    ("causal_d64", 1, 2, 2, 384, 384, 64, "and", [("causal",)], False, ("none",)),
    ("causal_alibi_d64_ragged", 2, 2, 2, 300, 300, 64, "and", [("causal",)], False, "alibi"),
    ("swa_softcap_d128_ragged", 1, 2, 2, 520, 520, 128, "and", [("causal",), ("sliding", 100)], False,
     ("softcap", 30.0)),
    ("doc_gqa_d128", 1, 4, 2, 700, 700, 128, "and", [("causal",), ("document",)], True, ("none",)),
    ("causal_bias_d64", 1, 2, 2, 333, 333, 64, "and", [("causal",)], False, "bias"),
    ("bias_softcap_d128", 1, 2, 1, 260, 390, 128, "and", [("causal",), ("sliding", 200)], False, "bias_softcap"),
    ("prefix_or_causal_d64", 1, 2, 2, 400, 400, 64, "or", [("prefix", 150), ("causal",)], False, ("none",)),
    ("cross_len_d64", 2, 2, 2, 200, 450, 64, "and", [("causal",)], False, ("none",)),
    ("cross_len_rev_d128", 1, 2, 2, 450, 200, 128, "or", [("sliding", 60), ("prefix", 20)], False, "alibi"),
    ("nomask_gqa_d64", 1, 4, 1, 256, 256, 64, "and", [], False, ("none",)),
    ("softcap_far_d64", 1, 2, 2, 256, 256, 64, "and", [("causal",)], False, ("softcap", 2.0)),
    ("tiny_1x1_d64", 1, 1, 1, 1, 1, 64, "and", [("causal",)], False, ("none",)),
    # D = 64 runs overlapped tiles and the dQ epilogue warps: documents with GQA
    # (partial tiles at every boundary, several query heads per CTA) and the
    # combined score_mod on a ragged length
    ("doc_gqa_alibi_d64", 2, 4, 2, 500, 500, 64, "and", [("causal",), ("document",)], True, "alibi"),
    ("bias_softcap_d64_ragged", 1, 2, 2, 390, 390, 64, "and", [("causal",)], False, "bias_softcap"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_small_backward_parity(case):
    name, B, Hq, Hkv, ql, kl, D, op, leaves, use_doc, spec = case
    seed = zlib.crc32(name.encode()) % 1000
    q, k, v, do = _inputs(B, Hq, Hkv, ql, kl, D, seed)
    doc = _doc(B, max(ql, kl), seed) if use_doc else None
    score = _score(spec, B, Hq, ql, kl, seed)
    dq, dk, dv = run_gpu(q, k, v, do, op, leaves, doc, score, bmB=(B if use_doc else 1))
    rq, rk, rv = oracle.backward(q, k, v, do, op, leaves, doc, score=score)
    for got, ref, nm in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        assert_grad_close(got, ref, f"{name} {nm}")
    assert _fa().device_status() == 0


def test_backward_without_the_split():
    """The unsplit BlockMask (every listed tile masked per element) gives the same gradients."""
    q, k, v, do = _inputs(1, 2, 2, 384, 384, 64, 31)
    rq, rk, rv = oracle.backward(q, k, v, do, "and", [("causal",)], None)
    dq, dk, dv = run_gpu(q, k, v, do, "and", [("causal",)], None, ("none",), split_full=False)
    for got, ref, nm in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        assert_grad_close(got, ref, f"unsplit {nm}")


def test_fully_masked_rows_and_unattended_keys():
    """kv >= q + 5 AND kv < 200: late query rows admit nothing (their dQ is 0) and
    keys >= 200 are attended by nobody (their dK and dV are 0)."""
    q, k, v, do = _inputs(1, 1, 1, 300, 300, 64, 32)
    leaves = [("sliding", -5), ("prefix", 200)]
    dq, dk, dv = run_gpu(q, k, v, do, "and", leaves, None, ("none",))
    rq, rk, rv = oracle.backward(q, k, v, do, "and", leaves, None)
    for got, ref, nm in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        assert_grad_close(got, ref, f"masked rows {nm}")
    assert torch.all(dk[0, 0, 200:] == 0) and torch.all(dv[0, 0, 200:] == 0)
    assert torch.all(dq[0, 0, 195:] == 0)


@pytest.mark.parametrize("ci", [0, 1, 4], ids=[W.CONFIGS[i].name for i in (0, 1, 4)])
def test_config_backward_parity(ci):
    """Configurations at full size: every gradient entry of two kv heads (and of the
    query heads that read them) against the oracle."""
    w = W.config(ci)
    q, k, v = W.qkv(w)
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(100 + ci)).to(torch.bfloat16)
    doc = W.document_ids(w)
    score = {"alibi": ("alibi", W.alibi_slopes(w.Hq)), "bias": ("bias", W.bias(w, 0)) if w.score == "bias" else None,
             "softcap": ("softcap", w.softcap), "none": ("none",)}[w.score]
    Bm = w.B if w.has_document else 1
    dq, dk, dv = run_gpu(q, k, v, do, w.mask_op, list(w.mask_leaves), doc, score, bmB=Bm)
    units = sorted({(0, 0), (w.B - 1, w.Hkv - 1)})
    rq, rk, rv = oracle.backward(q, k, v, do, w.mask_op, list(w.mask_leaves), doc, score=score, units=units)
    G = w.Hq // w.Hkv
    for b, hk in units:
        assert_grad_close(dk[b, hk], rk[b, hk], f"{w.name} dk[{b},{hk}]")
        assert_grad_close(dv[b, hk], rv[b, hk], f"{w.name} dv[{b},{hk}]")
        for hq in range(hk * G, hk * G + G):
            assert_grad_close(dq[b, hq], rq[b, hq], f"{w.name} dq[{b},{hq}]")
    assert _fa().device_status() == 0


@pytest.mark.parametrize("D", [64, 128])
def test_persistent_units_with_gqa_and_unattended_blocks(D):
    """(batch, kv head, kv block) units: 160 here, more than there are SMs (at D = 64
    persistent CTAs take several units in turn; at D = 128 a CTA runs each unit),
    with four query heads per kv head and (causal, q_len < kv_len) units that no
    query block attends to, whose dK, dV must be exactly zero."""
    B, Hq, Hkv, ql, kl = 4, 8, 2, 1536, 2560
    q, k, v, do = _inputs(B, Hq, Hkv, ql, kl, D, 321)
    score = ("alibi", W.alibi_slopes(Hq))
    dq, dk, dv = run_gpu(q, k, v, do, "and", [("causal",)], None, score)
    units = [(0, 0), (B - 1, Hkv - 1)]
    rq, rk, rv = oracle.backward(q, k, v, do, "and", [("causal",)], None, score=score, units=units)
    G = Hq // Hkv
    for b, hk in units:
        assert_grad_close(dk[b, hk], rk[b, hk], f"dk[{b},{hk}]")
        assert_grad_close(dv[b, hk], rv[b, hk], f"dv[{b},{hk}]")
        for hq in range(hk * G, hk * G + G):
            assert_grad_close(dq[b, hq], rq[b, hq], f"dq[{b},{hq}]")
    # keys past the last query position are attended by no query
    assert torch.all(dk[:, :, ql:] == 0) and torch.all(dv[:, :, ql:] == 0)
    assert _fa().device_status() == 0


@pytest.mark.parametrize("ci", [2, 3], ids=[W.CONFIGS[i].name for i in (2, 3)])
def test_config_structure_backward_parity(ci):
    """The D = 128 configurations (window + soft-cap, GQA document) with their mask,
    score_mod and head layout at S = 2048 (the full sizes are too slow for the
    dense fp64 oracle's backward), every gradient entry."""
    w = W.config(ci)
    S = 2048
    q, k, v, do = _inputs(1, w.Hq // (2 if w.Hkv < w.Hq else 8), max(1, w.Hkv // 4) if w.Hkv < w.Hq else 2,
                          S, S, w.D, 200 + ci)
    doc = None
    if w.has_document:
        doc = W.document_ids_from_lengths(W.document_lengths(S, w.doc_seed)).unsqueeze(0)
    score = ("softcap", w.softcap) if w.score == "softcap" else ("none",)
    dq, dk, dv = run_gpu(q, k, v, do, w.mask_op, list(w.mask_leaves), doc, score)
    rq, rk, rv = oracle.backward(q, k, v, do, w.mask_op, list(w.mask_leaves), doc, score=score)
    for got, ref, nm in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        assert_grad_close(got, ref, f"{w.name} S={S} {nm}")


def test_autograd_function_matches_oracle():
    """flex_attention_autograd: out.backward(dO) fills q/k/v.grad through fa_backward."""
    fa = _fa()
    q, k, v, do = _inputs(1, 4, 2, 300, 300, 64, 33)
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, 300, 300, transposed=True)
    qd, kd, vd = (t.cuda().requires_grad_() for t in (q, k, v))
    out, lse = fa.flex_attention_autograd(qd, kd, vd, bm)
    out.backward(do.cuda())
    torch.cuda.synchronize()
    rq, rk, rv = oracle.backward(q, k, v, do, "and", [("causal",)], None)
    for got, ref, nm in ((qd.grad, rq, "dq"), (kd.grad, rk, "dk"), (vd.grad, rv, "dv")):
        assert_grad_close(got, ref, f"autograd {nm}")


def test_backward_with_query_offset():
    """Gradients of queries at positions q_offset + i (a continuation chunk after a
    cache) against the oracle."""
    fa = _fa()
    S, n = 600, 200
    q, k, v, do = _inputs(1, 4, 2, n, S, 64, 34)
    slopes = W.alibi_slopes(4)
    bm = fa.create_block_mask("and", [("causal",), ("sliding", 256)], 1, 1, n, S, transposed=True, q_offset=S - n)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.flex_attention(qd, kd, vd, bm, score_mod=("alibi", slopes.cuda()))
    dq, dk, dv = fa.flex_attention_backward(qd, kd, vd, o, lse, dod, bm, score_mod=("alibi", slopes.cuda()))
    torch.cuda.synchronize()
    # the oracle's backward: offset rows through its q_offset-aware forward definition
    rq, rk, rv = oracle.backward(q, k, v, do, "and", [("causal",), ("sliding", 256)], None, score=("alibi", slopes),
                                 q_offset=S - n)
    for got, ref, nm in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        assert_grad_close(got, ref, f"offset {nm}")

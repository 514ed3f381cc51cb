"""fa_forward on the GPU against the fp64 oracle, element by element, within the
stated tolerances (O 2e-2 abs / 1e-2 rel, LSE 1e-3)."""

import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from helpers import assert_forward_close, block_mask_extents, gpu_score, workload_inputs

pytestmark = pytest.mark.gpu


def _fa():
    import block_sparse_attention_48_b200 as fa
    return fa


def _qkv(B, Hq, Hkv, ql, kl, D, seed, q_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn((B, Hq, ql, D), generator=g) * q_scale).to(torch.bfloat16)
    k = torch.randn((B, Hkv, kl, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, kl, D), generator=g).to(torch.bfloat16)
    return q, k, v


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


def _run(q, k, v, op, leaves, doc, score, bmB=1, bmH=1, scale=None):
    fa = _fa()
    dev = "cuda"
    bm = fa.create_block_mask(op, leaves, bmB, bmH, q.shape[2], k.shape[2], doc_ids=doc)
    o, lse = fa.flex_attention(q.to(dev), k.to(dev), v.to(dev), bm, score_mod=gpu_score(score), scale=scale)
    torch.cuda.synchronize()
    return o, lse


SMALL = [
    # name, B, Hq, Hkv, q_len, kv_len, D, op, leaves, doc, score
    ("causal_d64_ragged", 2, 2, 2, 300, 300, 64, "and", [("causal",)], False, ("none",)),
    ("causal_alibi_d64", 1, 4, 4, 384, 384, 64, "and", [("causal",)], False, "alibi"),
    ("swa_softcap_d128", 1, 2, 2, 520, 520, 128, "and", [("causal",), ("sliding", 100)], False, ("softcap", 30.0)),
    ("doc_gqa_d128", 1, 4, 2, 700, 700, 128, "and", [("causal",), ("document",)], True, ("none",)),
    ("causal_bias_d64", 1, 2, 2, 333, 333, 64, "and", [("causal",)], False, "bias"),
    ("nomask_d128", 1, 2, 1, 256, 256, 128, "and", [], False, ("none",)),
    ("prefix_or_causal_d64", 1, 2, 2, 400, 400, 64, "or", [("prefix", 150), ("causal",)], False, ("none",)),
    ("cross_len_d64", 2, 2, 2, 200, 450, 64, "and", [("causal",)], False, ("none",)),
    ("cross_len_rev_d128", 1, 2, 2, 450, 200, 128, "or", [("sliding", 60), ("prefix", 20)], False, "alibi"),
    ("doc_bias_d64", 2, 2, 1, 500, 500, 64, "and", [("causal",), ("document",)], True, "bias"),
    ("alibi_d128", 1, 2, 2, 260, 260, 128, "and", [("causal",)], False, "alibi"),
    ("softcap_d64", 1, 2, 2, 300, 300, 64, "and", [("causal",)], False, ("softcap", 20.0)),
    ("bias_d128_ragged", 1, 2, 2, 200, 330, 128, "and", [("causal",), ("sliding", 150)], False, "bias"),
    ("tiny_1x1", 1, 1, 1, 1, 1, 64, "and", [("causal",)], False, ("none",)),
    ("bias_softcap_d64", 2, 2, 2, 333, 333, 64, "and", [("causal",)], False, "bias_softcap"),
    ("bias_softcap_d128_ragged", 1, 4, 2, 270, 390, 128, "and", [("causal",), ("sliding", 200)], False,
     "bias_softcap"),
]


def _score_inputs(spec, B, Hq, ql, kl, seed):
    if spec == "alibi":
        return ("alibi", W.alibi_slopes(Hq))
    if spec == "bias":
        g = torch.Generator().manual_seed(seed + 99)
        return ("bias", torch.randn((B, Hq, ql, kl), generator=g).to(torch.bfloat16))
    if spec == "bias_softcap":
        # biases of N(0, 3) against cap 4: both tanh branches (|u| above and below 0.625)
        g = torch.Generator().manual_seed(seed + 98)
        return ("bias_softcap", (3 * torch.randn((B, Hq, ql, kl), generator=g)).to(torch.bfloat16), 4.0)
    return spec


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_parity(case):
    name, B, Hq, Hkv, ql, kl, D, op, leaves, use_doc, spec = case
    seed = zlib.crc32(name.encode()) % 1000
    q, k, v = _qkv(B, Hq, Hkv, ql, kl, D, seed)
    doc = _doc(B, max(ql, kl), seed) if use_doc else None
    score = _score_inputs(spec, B, Hq, ql, kl, seed)
    o, lse = _run(q, k, v, op, leaves, doc, score, bmB=(B if use_doc else 1))
    o_ref, lse_ref = oracle.forward(q, k, v, op, leaves, doc, score=score)
    assert_forward_close(o, lse, o_ref, lse_ref, name)


def config_parity_rows(w: W.Workload, ci: int, doc) -> torch.Tensor:
    """Rows (b, hq, q) compared at full size, deduplicated:
    - 192 seeded random rows;
    - every row of the first and the last query block of heads (0, 0) and (B-1, Hq-1);
    - with a document leaf, every row within 2 positions of each document boundary
      (where the document leaf cuts tiles into partial ones), for both heads;
    - every row of head (B-1, Hq-1), and with GQA also of head (0, 0), which reads
      another kv head."""
    heads = [(0, 0), (w.B - 1, w.Hq - 1)]
    rows = {tuple(r) for r in W.random_rows(w, 192, seed=ci).tolist()}
    for b, h in heads:
        for qi in list(range(0, min(128, w.q_len))) + list(range(max(0, w.q_len - 128), w.q_len)):
            rows.add((b, h, qi))
    if doc is not None:
        for b, h in heads:
            ids = doc[b, :w.q_len]
            starts = (torch.nonzero(ids[1:] != ids[:-1]).flatten() + 1).tolist()
            for s0 in starts:
                for qi in range(s0 - 2, s0 + 3):
                    if 0 <= qi < w.q_len:
                        rows.add((b, h, qi))
    whole = [(w.B - 1, w.Hq - 1)] + ([(0, 0)] if w.Hkv < w.Hq else [])
    for b, h in whole:
        for qi in range(w.q_len):
            rows.add((b, h, qi))
    return torch.tensor(sorted(rows), dtype=torch.int64)


@pytest.mark.parametrize("ci", range(len(W.CONFIGS)), ids=[c.name for c in W.CONFIGS])
def test_config_parity(ci):
    """Every configuration at full size, in the launch configuration the benchmark
    times, element by element against the oracle: all rows of the small
    configuration; for the others the rows of config_parity_rows (first and last
    query blocks, document boundaries, whole heads, random rows)."""
    w = W.config(ci)
    q, k, v, doc, score = workload_inputs(w)
    Bm, Hm = block_mask_extents(w)
    o, lse = _run(q, k, v, w.mask_op, list(w.mask_leaves), doc, score, bmB=Bm, bmH=Hm)
    if ci == 0:
        o_ref, lse_ref = oracle.forward(q, k, v, w.mask_op, list(w.mask_leaves), doc, score=score)
        assert_forward_close(o, lse, o_ref, lse_ref, w.name)
        return
    rows = config_parity_rows(w, ci, doc)
    o_ref, lse_ref = oracle.forward(q, k, v, w.mask_op, list(w.mask_leaves), doc, score=score, rows=rows)
    r = rows.numpy()
    o_s = o.float().cpu().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    l_s = lse.cpu().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    assert_forward_close(o_s, l_s, o_ref, lse_ref, f"{w.name} ({len(r)} rows)")
    assert _fa().device_status() == 0


def test_kv_len_zero_gives_zero_and_neg_inf():
    q, k, v = _qkv(1, 2, 2, 200, 0, 64, 1)
    o, lse = _run(q, k, v, "and", [("causal",)], None, ("none",))
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_fully_masked_rows():
    """causal AND (q - kv <= -1) admits nothing: O = 0, LSE = -inf everywhere."""
    q, k, v = _qkv(1, 2, 2, 300, 300, 128, 2)
    o, lse = _run(q, k, v, "and", [("causal",), ("sliding", -1)], None, ("none",))
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_partly_masked_rows_in_partial_tiles():
    """Rows with no admitted key inside otherwise non-empty tiles get O = 0 and
    LSE = -inf; the other rows of the same tiles are unaffected."""
    q, k, v = _qkv(1, 1, 1, 300, 300, 64, 3)
    # kv >= q + 5 AND kv < 200: rows q >= 195 admit nothing, earlier rows do
    leaves = [("sliding", -5), ("prefix", 200)]
    o, lse = _run(q, k, v, "and", leaves, None, ("none",))
    o_ref, lse_ref = oracle.forward(q, k, v, "and", leaves, None)
    assert_forward_close(o, lse, o_ref, lse_ref, "partly masked")


def test_value_ones_give_ones():
    q, k, v = _qkv(1, 2, 2, 384, 384, 64, 4)
    v = torch.ones_like(v)
    o, lse = _run(q, k, v, "and", [("causal",)], None, ("alibi", W.alibi_slopes(2)))
    assert (o.float() - 1).abs().max().item() <= 1e-2


def test_alibi_steep_and_negative_slopes():
    """ALiBi slopes of either sign, including ones too steep for the kernel's
    per-chunk bound of the row maximum (the column term is then applied before
    the maximum), with and without a causal mask."""
    q, k, v = _qkv(1, 4, 4, 384, 384, 64, 10)
    slopes = torch.tensor([3.0, -0.9, 0.5, 0.01], dtype=torch.float32)
    for leaves in ([("causal",)], []):
        o, lse = _run(q, k, v, "and", leaves, None, ("alibi", slopes))
        o_ref, lse_ref = oracle.forward(q, k, v, "and", leaves, None, score=("alibi", slopes))
        assert_forward_close(o, lse, o_ref, lse_ref, f"alibi steep {leaves}")


def test_mask_as_score_identity_on_gpu():
    """The causal BlockMask run equals an all-attend BlockMask with a 0 / -inf bias
    ("Concepts": a mask_mod is a score_mod returning -inf); bit equality reported."""
    S, D = 384, 64
    q, k, v = _qkv(1, 2, 2, S, S, D, 5)
    o1, l1 = _run(q, k, v, "and", [("causal",)], None, ("none",))
    keep = torch.tril(torch.ones(S, S, dtype=torch.bool))
    bias = torch.zeros((1, 2, S, S), dtype=torch.bfloat16).masked_fill(~keep, float("-inf"))
    o2, l2 = _run(q, k, v, "and", [], None, ("bias", bias))
    assert_forward_close(o1, l1, o2.double().cpu().numpy(), l2.double().cpu().numpy(), "mask-as-score")
    o_ref, lse_ref = oracle.forward(q, k, v, "and", [("causal",)], None)
    assert_forward_close(o2, l2, o_ref, lse_ref, "bias route vs oracle")
    print("mask-as-score bitwise equal:", bool(torch.equal(o1, o2)))


def test_bias_changes_every_call_without_rebuild():
    """attention-gym issue "Dynamic Bias Tensor": a new bias tensor on every call,
    same BlockMask, both results exact."""
    fa = _fa()
    S, D = 300, 64
    q, k, v = _qkv(1, 2, 2, S, S, D, 6)
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, S, S)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    for call in range(2):
        g = torch.Generator().manual_seed(100 + call)
        bias = torch.randn((1, 2, S, S), generator=g).to(torch.bfloat16)
        o, lse = fa.flex_attention(qd, kd, vd, bm, score_mod=("bias", bias.cuda()))
        torch.cuda.synchronize()
        o_ref, lse_ref = oracle.forward(q, k, v, "and", [("causal",)], None, score=("bias", bias))
        assert_forward_close(o, lse, o_ref, lse_ref, f"bias call {call}")


def test_softcap_far_branch():
    """Scores far beyond the polynomial range (|s| / cap > 0.625) exercise the
    exponential branch of tanh."""
    q, k, v = _qkv(1, 2, 2, 256, 256, 128, 7, q_scale=12.0)
    o, lse = _run(q, k, v, "and", [("causal",)], None, ("softcap", 30.0))
    o_ref, lse_ref = oracle.forward(q, k, v, "and", [("causal",)], None, score=("softcap", 30.0))
    assert_forward_close(o, lse, o_ref, lse_ref, "softcap far")


def test_explicit_scale_and_strided_layout():
    """[B, S, H, D] storage viewed as [B, H, S, D] (non-contiguous strides) and an
    explicit scale."""
    fa = _fa()
    B, H, S, D = 1, 2, 260, 64
    g = torch.Generator().manual_seed(8)
    base = [torch.randn((B, S, H, D), generator=g).to(torch.bfloat16) for _ in range(3)]
    q, k, v = [t.permute(0, 2, 1, 3) for t in base]
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, S, S)
    o, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, scale=0.05)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.forward(q.contiguous(), k.contiguous(), v.contiguous(), "and", [("causal",)], None,
                                    scale=0.05)
    assert_forward_close(o, lse, o_ref, lse_ref, "strided")


def test_blockmask_broadcast_over_heads_and_batch():
    """A BlockMask with B = H = 1 serves every (b, h); one with H = Hq is equivalent."""
    fa = _fa()
    q, k, v = _qkv(2, 4, 4, 300, 300, 64, 9)
    o1, _ = _run(q, k, v, "and", [("causal",)], None, ("none",), bmB=1, bmH=1)
    o2, _ = _run(q, k, v, "and", [("causal",)], None, ("none",), bmB=2, bmH=4)
    assert torch.equal(o1, o2)


def test_bias_broadcast_over_batch_and_heads():
    """A bias expanded from [1, 1, Sq, Skv] (stride 0 over batch and heads) is read
    as one plane for every (b, h); one expanded over heads only likewise."""
    fa = _fa()
    B, H, S, D = 2, 3, 300, 64
    q, k, v = _qkv(B, H, H, S, S, D, 11)
    g = torch.Generator().manual_seed(12)
    plane = torch.randn((1, 1, S, S), generator=g).to(torch.bfloat16)
    per_b = torch.randn((B, 1, S, S), generator=g).to(torch.bfloat16)
    for bias in (plane.expand(B, H, S, S), per_b.expand(B, H, S, S)):
        bm = fa.create_block_mask("and", [("causal",)], 1, 1, S, S)
        o, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, score_mod=("bias", bias.cuda()))
        torch.cuda.synchronize()
        o_ref, lse_ref = oracle.forward(q, k, v, "and", [("causal",)], None, score=("bias", bias.contiguous()))
        assert_forward_close(o, lse, o_ref, lse_ref, f"bias broadcast {tuple(bias.stride())}")


def test_expanded_kv_heads_are_materialised():
    """K / V expanded over heads (stride 0) are copied by the binding before the
    call; the result matches the oracle on the materialised tensors."""
    fa = _fa()
    B, H, S, D = 1, 4, 260, 128
    q, k, v = _qkv(B, H, 1, S, S, D, 13)
    ke, ve = k.expand(B, H, S, D), v.expand(B, H, S, D)
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, S, S)
    o, lse = fa.flex_attention(q.cuda(), ke.cuda(), ve.cuda(), bm)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.forward(q, ke.contiguous(), ve.contiguous(), "and", [("causal",)], None)
    assert_forward_close(o, lse, o_ref, lse_ref, "expanded kv")
    with pytest.raises(TypeError):
        fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, out=torch.empty((B, 1, S, D), dtype=torch.bfloat16,
                                                                            device="cuda").expand(B, H, S, D))


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2, reason="one device")
def test_forward_on_second_device():
    """Launch set-up is per context: a forward on device 1 after device 0 works."""
    fa = _fa()
    q, k, v = _qkv(1, 2, 2, 300, 300, 64, 14)
    for dev in (0, 1):
        with torch.cuda.device(dev):
            bm = fa.create_block_mask("and", [("causal",)], 1, 1, 300, 300, device=torch.device("cuda", dev))
            o, lse = fa.flex_attention(q.to(f"cuda:{dev}"), k.to(f"cuda:{dev}"), v.to(f"cuda:{dev}"), bm)
            torch.cuda.synchronize(dev)
        o_ref, lse_ref = oracle.forward(q, k, v, "and", [("causal",)], None)
        assert_forward_close(o, lse, o_ref, lse_ref, f"device {dev}")


@pytest.mark.parametrize("ci", [0, 1, 2, 4], ids=[W.CONFIGS[i].name for i in (0, 1, 2, 4)])
def test_unsplit_block_mask_forward(ci):
    """Without the full / partial split every listed tile is masked per element;
    the result is the same attention (sampled rows at full size)."""
    w = W.config(ci)
    q, k, v, doc, score = workload_inputs(w)
    fa = _fa()
    bm = fa.create_block_mask(w.mask_op, list(w.mask_leaves), 1, 1, w.q_len, w.kv_len, split_full=False)
    assert bm.desc.has_full == 0
    o, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, score_mod=gpu_score(score))
    torch.cuda.synchronize()
    rows = W.random_rows(w, 256, seed=50 + ci)
    o_ref, lse_ref = oracle.forward(q, k, v, w.mask_op, list(w.mask_leaves), doc, score=score, rows=rows)
    r = rows.numpy()
    assert_forward_close(o.float().cpu().numpy()[r[:, 0], r[:, 1], r[:, 2]], lse.cpu().numpy()[r[:, 0], r[:, 1], r[:, 2]],
                         o_ref, lse_ref, f"unsplit {w.name}")
    assert fa.device_status() == 0


def test_device_status_clean():
    assert _fa().device_status() == 0


def _paged_cache(k, v, seed, extra=5, share_first=False):
    """Scatter K, V [B, Hkv, S, D] into page pools by a seeded permutation (plus
    unused noise pages); optionally batch 1 reuses batch 0's first page."""
    B, H, S, D = k.shape
    nkv = -(-S // 128)
    g = torch.Generator().manual_seed(seed)
    P = B * nkv + extra
    kp = torch.randn((P, H, 128, D), generator=g).to(torch.bfloat16)
    vp = torch.randn((P, H, 128, D), generator=g).to(torch.bfloat16)
    pt = torch.randperm(P, generator=g)[: B * nkv].view(B, nkv).to(torch.int32)
    if share_first and B > 1:
        pt[1, 0] = pt[0, 0]
    for b in range(B):
        for kb in range(nkv):
            if share_first and b == 1 and kb == 0:
                continue
            n = min(128, S - 128 * kb)
            kp[pt[b, kb], :, :n] = k[b, :, 128 * kb: 128 * kb + n]
            vp[pt[b, kb], :, :n] = v[b, :, 128 * kb: 128 * kb + n]
    # a padded page table row (stride > nkv)
    ptp = torch.full((B, nkv + 3), -7, dtype=torch.int32)
    ptp[:, :nkv] = pt
    return kp, vp, ptp


PAGED = [
    ("paged_causal_alibi_d64_ragged", 2, 4, 2, 300, 64, "and", [("causal",)], "alibi", False),
    ("paged_swa_softcap_d128", 1, 2, 2, 520, 128, "and", [("causal",), ("sliding", 100)], ("softcap", 30.0), False),
    ("paged_shared_prefix_d64", 2, 2, 1, 384, 64, "or", [("prefix", 128), ("causal",)], ("none",), True),
]


@pytest.mark.parametrize("case", PAGED, ids=[c[0] for c in PAGED])
def test_paged_forward_parity(case):
    """fa_forward_paged against the oracle on the gathered logical K, V (paper
    review sec. 4.5: the BlockMask's kv indices as a page table)."""
    fa = _fa()
    name, B, Hq, Hkv, S, D, op, leaves, spec, share = case
    seed = zlib.crc32(name.encode()) % 1000
    q, k, v = _qkv(B, Hq, Hkv, S, S, D, seed)
    if share:  # sequences with a common first page: equal first keys and values
        k[1, :, :128] = k[0, :, :128]
        v[1, :, :128] = v[0, :, :128]
    kp, vp, pt = _paged_cache(k, v, seed, share_first=share)
    score = _score_inputs(spec, B, Hq, S, S, seed)
    bm = fa.create_block_mask(op, leaves, 1, 1, S, S)
    o, lse = fa.flex_attention_paged(q.cuda(), kp.cuda(), vp.cuda(), pt.cuda(), bm, score_mod=gpu_score(score))
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    o_ref, lse_ref = oracle.forward_paged(q, kp, vp, pt, S, op, leaves, None, score=score)
    assert_forward_close(o, lse, o_ref, lse_ref, name)
    # and the contiguous path on the same logical tensors agrees
    o2, lse2 = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, score_mod=gpu_score(score))
    assert_forward_close(o, lse, o2.double().cpu().numpy(), lse2.double().cpu().numpy(), f"{name} vs contiguous")


def test_paged_headline_shape():
    """The headline workload's shape (B4 H16 S2048 D64, causal + ALiBi) over a
    randomly permuted page pool: sampled rows against the oracle."""
    fa = _fa()
    w = W.config(1)
    q, k, v = W.qkv(w)
    kp, vp, pt = _paged_cache(k, v, 77)
    slopes = W.alibi_slopes(w.Hq)
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, w.q_len, w.kv_len)
    o, lse = fa.flex_attention_paged(q.cuda(), kp.cuda(), vp.cuda(), pt.cuda(), bm, score_mod=("alibi", slopes.cuda()))
    torch.cuda.synchronize()
    rows = W.random_rows(w, 384, seed=78)
    o_ref, lse_ref = oracle.forward_paged(q, kp, vp, pt, w.kv_len, "and", [("causal",)], None,
                                          score=("alibi", slopes), rows=rows)
    r = rows.numpy()
    assert_forward_close(o.float().cpu().numpy()[r[:, 0], r[:, 1], r[:, 2]], lse.cpu().numpy()[r[:, 0], r[:, 1], r[:, 2]],
                         o_ref, lse_ref, "paged headline")


def test_paged_bad_page_is_reported_without_fault():
    """A page entry outside the pool is clamped in the kernel and reported."""
    fa = _fa()
    q, k, v = _qkv(1, 2, 2, 256, 256, 64, 79)
    kp, vp, pt = _paged_cache(k, v, 80)
    pt[0, 1] = kp.shape[0] + 50
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, 256, 256)
    fa.flex_attention_paged(q.cuda(), kp.cuda(), vp.cuda(), pt.cuda(), bm)
    assert fa.device_status() == fa.FA_ERR_BAD_BLOCKMASK
    assert fa.device_status() == 0


@pytest.mark.parametrize("op,leaves,spec,D,n", [
    ("and", [("causal",)], "alibi", 64, 1),
    ("and", [("causal",), ("sliding", 300)], ("softcap", 30.0), 128, 3),
    ("and", [("causal",), ("document",)], ("none",), 128, 130),
])
def test_query_offset_rows(op, leaves, spec, D, n):
    """Queries at positions q_offset + i (a decoding step, or a continuation after a
    cache): BlockMask bit-exact and the forward pass within tolerance of the oracle."""
    fa = _fa()
    S, Hq, Hkv = 700, 4, 2
    q, k, v = _qkv(1, Hq, Hkv, n, S, D, 90 + n)
    off = S - n
    doc = _doc(1, S, 91) if any(l[0] == "document" for l in leaves) else None
    score = _score_inputs(spec, 1, Hq, n, S, 92)
    bm = fa.create_block_mask(op, leaves, 1, 1, n, S, doc_ids=doc, q_offset=off)
    torch.cuda.synchronize()
    ref_bm = oracle.block_mask(op, leaves, doc, 1, 1, n, S, q_offset=off)
    from helpers import block_mask_equal
    block_mask_equal(bm.to_cpu(), ref_bm)
    o, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, score_mod=gpu_score(score))
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.forward(q, k, v, op, leaves, doc, score=score, q_offset=off)
    assert_forward_close(o, lse, o_ref, lse_ref, f"offset {off}")

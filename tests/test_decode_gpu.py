"""fa_decode (FlexDecoding: a few query tokens against a long cache, split along
KV and merged) against the fp64 oracle with the queries at their positions
(q_offset), within the forward pass's tolerances."""

import zlib

import pytest
import torch

import oracle
import workloads as W
from helpers import assert_forward_close, gpu_score

pytestmark = pytest.mark.gpu


def _fa():
    import block_sparse_attention_48_b200 as fa
    return fa


def _inputs(B, Hq, Hkv, ql, kl, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, ql, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, kl, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, kl, D), generator=g).to(torch.bfloat16)
    return q, k, v


def _doc(B, L, seed):
    g = torch.Generator().manual_seed(seed)
    rows = []
    for b in range(B):
        lengths, acc = [], 0
        while acc < L:
            n = int(torch.randint(100, 1500, (1,), generator=g))
            lengths.append(min(n, L - acc))
            acc += lengths[-1]
        rows.append(W.document_ids_from_lengths(lengths))
    return torch.stack(rows)


CASES = [
    # name, B, Hq, Hkv, q_len, kv_len, D, op, leaves, doc, score
    ("gqa4_causal_d128", 2, 8, 2, 1, 3000, 128, "and", [("causal",)], False, ("none",)),
    ("mha_window_alibi_d64", 3, 4, 4, 4, 1000, 64, "and", [("causal",), ("sliding", 256)], False, "alibi"),
    ("gqa8_doc_softcap_d128", 1, 16, 2, 2, 5000, 128, "and", [("causal",), ("document",)], True, ("softcap", 30.0)),
    ("prefix_or_causal_bias_d64", 2, 2, 1, 1, 777, 64, "or", [("prefix", 300), ("causal",)], False, "bias"),
    ("bias_softcap_d128", 1, 4, 2, 3, 640, 128, "and", [("causal",)], False, "bias_softcap"),
    ("one_block_d64", 2, 4, 1, 1, 100, 64, "and", [("causal",)], False, ("none",)),
    ("long_d64_gqa16", 1, 16, 1, 1, 20000, 64, "and", [("causal",)], False, ("none",)),
]


def _score(spec, B, Hq, ql, kl, seed):
    g = torch.Generator().manual_seed(seed + 5)
    if spec == "alibi":
        return ("alibi", W.alibi_slopes(Hq))
    if spec == "bias":
        return ("bias", torch.randn((B, Hq, ql, kl), generator=g).to(torch.bfloat16))
    if spec == "bias_softcap":
        return ("bias_softcap", (3 * torch.randn((B, Hq, ql, kl), generator=g)).to(torch.bfloat16), 4.0)
    return spec


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_decode_parity(case):
    fa = _fa()
    name, B, Hq, Hkv, ql, kl, D, op, leaves, use_doc, spec = case
    seed = zlib.crc32(name.encode()) % 1000
    q, k, v = _inputs(B, Hq, Hkv, ql, kl, D, seed)
    off = kl - ql  # the new tokens are the last positions of each sequence
    doc = _doc(B, kl, seed) if use_doc else None
    score = _score(spec, B, Hq, ql, kl, seed)
    bm = fa.create_block_mask(op, leaves, B if use_doc else 1, 1, ql, kl, doc_ids=doc, q_offset=off)
    o, lse = fa.flex_decode(q.cuda(), k.cuda(), v.cuda(), bm, score_mod=gpu_score(score))
    torch.cuda.synchronize()
    assert fa.device_status(ws=fa.decode_workspace(torch.device("cuda", 0))) == 0
    o_ref, lse_ref = oracle.forward(q, k, v, op, leaves, doc, score=score, q_offset=off)
    assert_forward_close(o, lse, o_ref, lse_ref, name)
    # the prefill kernel on the same problem agrees
    o2, lse2 = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, score_mod=gpu_score(score))
    assert_forward_close(o, lse, o2.double().cpu().numpy(), lse2.double().cpu().numpy(), f"{name} vs forward")


def test_decode_empty_cache_and_unsupported_group():
    fa = _fa()
    q, k, v = _inputs(1, 4, 1, 1, 0, 64, 1)
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, 1, 0)
    o, lse = fa.flex_decode(q.cuda(), k.cuda(), v.cuda(), bm)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    q, k, v = _inputs(1, 32, 1, 1, 256, 64, 2)  # 32 query heads on one kv head: more than 16 rows
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, 1, 256, q_offset=255)
    with pytest.raises(fa.FlexAttnError):
        fa.flex_decode(q.cuda(), k.cuda(), v.cuda(), bm)


def test_decode_segments_of_unequal_length():
    """Per-batch document ids give every batch's BlockMask row its own length, and
    the list of (batch, kv head, block) work is shorter than the grid, so some
    CTAs' shares are empty and pieces of one segment sit on several CTAs."""
    fa = _fa()
    B, Hq, Hkv, ql, kl, D = 12, 4, 2, 1, 3000, 128
    q, k, v = _inputs(B, Hq, Hkv, ql, kl, D, 31)
    doc = _doc(B, kl, 32)
    off = kl - ql
    bm = fa.create_block_mask("and", [("causal",), ("document",)], B, 1, ql, kl, doc_ids=doc, q_offset=off)
    counts = (bm.kv_num_blocks + bm.full_kv_num_blocks).flatten().tolist()
    assert len(set(counts)) > 1
    o, lse = fa.flex_decode(q.cuda(), k.cuda(), v.cuda(), bm)
    torch.cuda.synchronize()
    assert fa.device_status(ws=fa.decode_workspace(torch.device("cuda", 0))) == 0
    o_ref, lse_ref = oracle.forward(q, k, v, "and", [("causal",), ("document",)], doc, q_offset=off)
    assert_forward_close(o, lse, o_ref, lse_ref, "unequal segments")


def test_decode_empty_rows_within_the_list():
    """BlockMask rows emptied for batches 1 and 3 (the BlockMask decides which
    blocks are read): those batches' rows are O = 0, LSE = -inf, and the
    segments around them are unaffected."""
    fa = _fa()
    B, Hq, Hkv, ql, kl, D = 5, 8, 2, 1, 2000, 64
    q, k, v = _inputs(B, Hq, Hkv, ql, kl, D, 41)
    off = kl - ql
    bm = fa.create_block_mask("and", [("causal",)], B, 1, ql, kl, q_offset=off)
    for b in (1, 3):
        bm.kv_num_blocks[b].zero_()
        bm.full_kv_num_blocks[b].zero_()
    o, lse = fa.flex_decode(q.cuda(), k.cuda(), v.cuda(), bm)
    torch.cuda.synchronize()
    assert fa.device_status(ws=fa.decode_workspace(torch.device("cuda", 0))) == 0
    o_ref, lse_ref = oracle.forward(q, k, v, "and", [("causal",)], None, q_offset=off)
    keep = [0, 2, 4]
    assert_forward_close(o[keep], lse[keep], o_ref[keep], lse_ref[keep], "rows around empty ones")
    for b in (1, 3):
        assert torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b]))


def test_decode_benchmark_workload_full_size():
    """The benchmark's decode workload at full size (B8 Hq32 Hkv8, one token at
    position 32767 against a 32k cache, D128, causal), every output row against
    the oracle."""
    fa = _fa()
    B, Hq, Hkv, ql, kl, D = 8, 32, 8, 1, 32768, 128
    q, k, v = _inputs(B, Hq, Hkv, ql, kl, D, 51)
    off = kl - ql
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, ql, kl, q_offset=off)
    o, lse = fa.flex_decode(q.cuda(), k.cuda(), v.cuda(), bm)
    torch.cuda.synchronize()
    assert fa.device_status(ws=fa.decode_workspace(torch.device("cuda", 0))) == 0
    o_ref, lse_ref = oracle.forward(q, k, v, "and", [("causal",)], None, q_offset=off)
    assert_forward_close(o, lse, o_ref, lse_ref, "decode workload, full size")


def test_decode_workspace_reused_across_calls_and_shapes():
    """The CTAs share out the kv blocks through counters in the workspace; every
    call leaves them ready for the next, so one zeroed workspace serves repeated
    calls and calls of another shape (each checked against the oracle)."""
    fa = _fa()
    lib = fa.library()
    shapes = [(4, 16, 4, 1, 9000, 128), (3, 8, 8, 2, 3000, 64)]
    need = max(int(lib.fa_decode_workspace_size(B, Hq, Hkv, ql, kl, D)) for B, Hq, Hkv, ql, kl, D in shapes)
    ws = torch.zeros((need,), dtype=torch.uint8, device="cuda")
    for i, (B, Hq, Hkv, ql, kl, D) in enumerate(shapes + shapes[:1]):
        q, k, v = _inputs(B, Hq, Hkv, ql, kl, D, 60 + i)
        off = kl - ql
        bm = fa.create_block_mask("and", [("causal",)], 1, 1, ql, kl, q_offset=off)
        o_ref, lse_ref = oracle.forward(q, k, v, "and", [("causal",)], None, q_offset=off)
        qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
        for rep in range(3):
            o, lse = fa.flex_decode(qc, kc, vc, bm, ws=ws)
            torch.cuda.synchronize()
            assert_forward_close(o, lse, o_ref, lse_ref, f"shape {i}, call {rep}")
        assert fa.device_status(ws=ws) == 0

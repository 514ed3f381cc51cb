"""fa_create_block_mask on the GPU against the oracle: bit-exact BlockMask tensors."""

import pytest
import torch

import oracle
import workloads as W
from helpers import block_mask_equal, block_mask_extents

pytestmark = pytest.mark.gpu


def _fa():
    import block_sparse_attention_48_b200 as fa
    return fa


@pytest.mark.parametrize("ci", range(len(W.CONFIGS)), ids=[c.name for c in W.CONFIGS])
def test_configs_bit_exact(ci):
    w = W.config(ci)
    doc = W.document_ids(w)
    Bm, Hm = block_mask_extents(w)
    bm = _fa().create_block_mask(w.mask_op, w.mask_leaves, Bm, Hm, w.q_len, w.kv_len, doc_ids=doc)
    torch.cuda.synchronize()
    ref = oracle.block_mask(w.mask_op, list(w.mask_leaves), doc, Bm, Hm, w.q_len, w.kv_len)
    block_mask_equal(bm.to_cpu(), ref)


@pytest.mark.parametrize("ci", range(len(W.CONFIGS)), ids=[c.name for c in W.CONFIGS])
def test_configs_unsplit_bit_exact(ci):
    """fa_create_block_mask_unsplit: every non-empty tile in kv_indices, full lists empty."""
    w = W.config(ci)
    doc = W.document_ids(w)
    Bm, Hm = block_mask_extents(w)
    bm = _fa().create_block_mask(w.mask_op, w.mask_leaves, Bm, Hm, w.q_len, w.kv_len, doc_ids=doc,
                                 split_full=False)
    torch.cuda.synchronize()
    ref = oracle.block_mask(w.mask_op, list(w.mask_leaves), doc, Bm, Hm, w.q_len, w.kv_len, split_full=False)
    block_mask_equal(bm.to_cpu(), ref)


def _random_doc(B, L, seed, shuffle=False):
    g = torch.Generator().manual_seed(seed)
    rows = []
    for b in range(B):
        lengths, acc = [], 0
        while acc < L:
            n = int(torch.randint(1, 300, (1,), generator=g))
            lengths.append(min(n, L - acc))
            acc += lengths[-1]
        ids = W.document_ids_from_lengths(lengths)
        if shuffle:  # ids not sorted: equal ids may sit in separate runs
            ids = ids % 3
        rows.append(ids)
    return torch.stack(rows)


CASES = [
    ("and", [("causal",)], 1, 1, 300, 300, None),
    ("and", [("causal",)], 1, 3, 384, 200, None),
    ("and", [("causal",), ("sliding", 37)], 1, 1, 1000, 1000, None),
    ("and", [("causal",), ("sliding", 300)], 1, 1, 640, 513, None),
    ("or", [("prefix", 90), ("causal",)], 1, 1, 520, 520, None),
    ("or", [("sliding", -200), ("prefix", 130)], 1, 1, 400, 700, None),
    ("and", [], 1, 1, 260, 130, None),
    ("and", [("causal",), ("document",)], 2, 1, 900, 900, "sorted"),
    ("and", [("document",)], 2, 2, 777, 777, "shuffled"),
    ("or", [("document",), ("causal",)], 1, 1, 600, 600, "shuffled"),
    ("and", [("causal",), ("sliding", 64), ("prefix", 1000)], 1, 1, 1100, 1100, None),
    ("and", [("causal",)], 1, 1, 256, 0, None),
    ("and", [("causal",)], 1, 1, 1, 1, None),
]


@pytest.mark.parametrize("op,leaves,B,H,ql,kl,doc", CASES)
def test_random_cases_bit_exact(op, leaves, B, H, ql, kl, doc):
    d = None
    if doc is not None:
        d = _random_doc(B, max(ql, kl), seed=ql + kl, shuffle=(doc == "shuffled"))
    bm = _fa().create_block_mask(op, leaves, B, H, ql, kl, doc_ids=d)
    torch.cuda.synchronize()
    ref = oracle.block_mask(op, leaves, d, B, H, ql, kl)
    block_mask_equal(bm.to_cpu(), ref)


def test_causal_closed_form_on_gpu():
    n = 16
    bm = _fa().create_block_mask("and", [("causal",)], 1, 1, 128 * n, 128 * n).to_cpu()
    for i in range(n):
        assert bm["full_kv_num_blocks"][0, 0, i] == i and bm["kv_num_blocks"][0, 0, i] == 1
        assert list(bm["full_kv_indices"][0, 0, i, :i]) == list(range(i))
        assert bm["kv_indices"][0, 0, i, 0] == i


def test_swapping_doc_layouts_needs_no_rebuild():
    """Two document layouts in one process, one after the other, both exact."""
    fa = _fa()
    for seed in (1, 2):
        d = _random_doc(1, 1500, seed)
        bm = fa.create_block_mask("and", [("causal",), ("document",)], 1, 1, 1500, 1500, doc_ids=d)
        torch.cuda.synchronize()
        block_mask_equal(bm.to_cpu(), oracle.block_mask("and", [("causal",), ("document",)], d, 1, 1, 1500, 1500))


@pytest.mark.parametrize("op,leaves,doc", [
    ("or", [("prefix", 200000), ("causal",)], None),
    ("and", [("document",)], "sorted"),
])
def test_long_kv_crosses_classification_chunks(op, leaves, doc):
    """More than 2048 kv blocks: the kernel classifies kv blocks in chunks."""
    ql, kl = 256, 2100 * 128 + 77
    d = _random_doc(1, kl, seed=11) if doc else None
    if d is not None:  # long documents, so that whole tiles fall inside one
        d = d // 40
    bm = _fa().create_block_mask(op, leaves, 1, 1, ql, kl, doc_ids=d)
    torch.cuda.synchronize()
    block_mask_equal(bm.to_cpu(), oracle.block_mask(op, leaves, d, 1, 1, ql, kl))


def _transposed_equal(got: dict, ref: dict):
    for key in ("q_num_blocks", "q_indices", "full_q_num_blocks", "full_q_indices"):
        a, b = got[key], ref[key]
        assert a.shape == b.shape, (key, a.shape, b.shape)
        if not (a == b).all():
            raise AssertionError(f"{key} differs at {(a != b).nonzero()}")


@pytest.mark.parametrize("ci", range(len(W.CONFIGS)), ids=[c.name for c in W.CONFIGS])
def test_configs_transposed_bit_exact(ci):
    """The transposed view ("used in backward") of every configuration."""
    w = W.config(ci)
    doc = W.document_ids(w)
    Bm, Hm = block_mask_extents(w)
    bm = _fa().create_block_mask(w.mask_op, w.mask_leaves, Bm, Hm, w.q_len, w.kv_len, doc_ids=doc, transposed=True)
    torch.cuda.synchronize()
    block_mask_equal(bm.to_cpu(), oracle.block_mask(w.mask_op, list(w.mask_leaves), doc, Bm, Hm, w.q_len, w.kv_len))
    _transposed_equal(bm.transposed_to_cpu(),
                      oracle.block_mask_transposed(w.mask_op, list(w.mask_leaves), doc, Bm, Hm, w.q_len, w.kv_len))


@pytest.mark.parametrize("op,leaves,B,H,ql,kl,doc", CASES)
def test_random_cases_transposed_bit_exact(op, leaves, B, H, ql, kl, doc):
    d = None
    if doc is not None:
        d = _random_doc(B, max(ql, kl), seed=ql + kl, shuffle=(doc == "shuffled"))
    bm = _fa().create_block_mask(op, leaves, B, H, ql, kl, doc_ids=d, transposed=True)
    torch.cuda.synchronize()
    _transposed_equal(bm.transposed_to_cpu(), oracle.block_mask_transposed(op, leaves, d, B, H, ql, kl))

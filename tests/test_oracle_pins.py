"""Pins for the CPU oracle: closed forms, brute force, library special cases and
invariants, so that a dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one test.  No GPU involved.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
CAUSAL = [("causal",)]


def bf(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def lists(bm, b=0, h=0):
    """(full lists, partial lists) per query block as python lists."""
    full, part = [], []
    for i in range(bm["kv_num_blocks"].shape[2]):
        nf = bm["full_kv_num_blocks"][b, h, i]
        npart = bm["kv_num_blocks"][b, h, i]
        full.append(list(bm["full_kv_indices"][b, h, i, :nf]))
        part.append(list(bm["kv_indices"][b, h, i, :npart]))
    return full, part


# ---------------------------------------------------------------- BlockMask pins

def test_golden_causal_blockmask_s256():
    """attention-gym "Concepts", BlockMask Internals: causal is the lower triangle."""
    want = {}
    with open(os.path.join(GOLDEN, "causal_blockmask_s256.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            qb, rest = line.split(":")
            full_s, part_s = rest.split()
            parse = lambda s: [int(x) for x in s.split("=")[1].split(",") if x]
            want[int(qb)] = (parse(full_s), parse(part_s))
    bm = oracle.block_mask("and", CAUSAL, None, 1, 1, 256, 256)
    full, part = lists(bm)
    for qb, (f, p) in want.items():
        assert full[qb] == f and part[qb] == p
    # every padded slot is 0
    assert bm["kv_indices"][0, 0, 0, 1] == 0 and bm["full_kv_indices"][0, 0, 0, 0] == 0


@pytest.mark.parametrize("n", [1, 2, 5, 16])
def test_causal_block_counts_closed_form(n):
    """Causal at S = 128 n: query block i has i full blocks (0..i-1), one partial
    block (i) and n-1-i empty ones; sparsity (n-1)/(2n)."""
    S = 128 * n
    bm = oracle.block_mask("and", CAUSAL, None, 1, 1, S, S)
    full, part = lists(bm)
    for i in range(n):
        assert full[i] == list(range(i))
        assert part[i] == [i]
    n_full = sum(len(f) for f in full)
    n_part = sum(len(p) for p in part)
    n_empty = n * n - n_full - n_part
    assert (n_full, n_part, n_empty) == (n * (n - 1) // 2, n, n * (n - 1) // 2)
    assert n_empty / (n * n) == pytest.approx((n - 1) / (2 * n))


def test_causal_sliding_block_counts_closed_form():
    """causal AND (q - kv <= 1024) at S = 8192: full = min(i, 7) blocks, partial =
    1 + [i >= 8] (the diagonal and block i-8); totals 420 / 120 / 3556."""
    n = 64
    bm = oracle.block_mask("and", [("causal",), ("sliding", 1024)], None, 1, 1, 128 * n, 128 * n)
    full, part = lists(bm)
    for i in range(n):
        assert full[i] == list(range(max(0, i - 7), i))
        assert part[i] == ([i - 8, i] if i >= 8 else [i])
    n_full = sum(len(f) for f in full)
    n_part = sum(len(p) for p in part)
    assert (n_full, n_part, n * n - n_full - n_part) == (420, 120, 3556)


def _torch_dense(kind, q_len, kv_len, **kw):
    """Masks built from library routines (tril/triu/block_diag), independent of the
    oracle's per-element predicates."""
    ones = torch.ones((q_len, kv_len), dtype=torch.bool)
    if kind == "causal":
        return torch.tril(ones)
    if kind == "causal_sliding":
        W_ = kw["W"]
        return torch.tril(ones) & torch.triu(ones, diagonal=-W_)
    if kind == "causal_doc":
        blocks = [torch.ones((n, n), dtype=torch.bool) for n in kw["lengths"]]
        return torch.tril(ones) & torch.block_diag(*blocks)[:q_len, :kv_len]
    if kind == "prefix_or_causal":
        m = torch.tril(ones).clone()
        m[:, : kw["P"]] = True
        return m
    raise KeyError(kind)


DENSE_CASES = [
    ("causal", "and", [("causal",)], {}),
    ("causal_sliding", "and", [("causal",), ("sliding", 37)], {"W": 37}),
    ("causal_doc", "and", [("causal",), ("document",)], {"lengths": [70, 5, 200, 1, 124]}),
    ("prefix_or_causal", "or", [("prefix", 90), ("causal",)], {"P": 90}),
]


@pytest.mark.parametrize("kind,op,leaves,kw", DENSE_CASES, ids=[c[0] for c in DENSE_CASES])
def test_dense_mask_matches_library_construction(kind, op, leaves, kw):
    S = 400
    doc = None
    if "lengths" in kw:
        doc = W.document_ids_from_lengths(kw["lengths"]).unsqueeze(0)
    got = oracle.dense_mask(op, leaves, doc, 0, 0, S, S)
    want = _torch_dense(kind, S, S, **kw).numpy()
    assert np.array_equal(got, want)


@pytest.mark.parametrize("kind,op,leaves,kw", DENSE_CASES, ids=[c[0] for c in DENSE_CASES])
@pytest.mark.parametrize("q_len,kv_len", [(256, 256), (300, 300), (384, 200), (130, 513)])
def test_block_classes_brute_force(kind, op, leaves, kw, q_len, kv_len):
    """Full / partial / empty from a brute-force count over each 128x128 tile of an
    independently built dense mask, in-range positions only."""
    doc = None
    if "lengths" in kw:
        lengths = kw["lengths"] + [max(q_len, kv_len)]
        doc = W.document_ids_from_lengths(lengths)[: max(q_len, kv_len)].unsqueeze(0)
        kw = dict(kw, lengths=lengths)
    dense = _torch_dense(kind, max(q_len, kv_len), max(q_len, kv_len), **kw)[:q_len, :kv_len].numpy()
    bm = oracle.block_mask(op, leaves, doc, 1, 1, q_len, kv_len)
    full, part = lists(bm)
    nq, nkv = -(-q_len // 128), -(-kv_len // 128)
    for i in range(nq):
        want_full, want_part = [], []
        for j in range(nkv):
            tile = dense[128 * i: 128 * (i + 1), 128 * j: 128 * (j + 1)]
            c = int(tile.sum())
            if c == tile.size:
                want_full.append(j)
            elif c > 0:
                want_part.append(j)
        assert full[i] == want_full, (i, full[i], want_full)
        assert part[i] == want_part, (i, part[i], want_part)
    # without the split every non-empty tile is a listed (masked) tile
    uf, up = lists(oracle.block_mask(op, leaves, doc, 1, 1, q_len, kv_len, split_full=False))
    for i in range(nq):
        tiles = [dense[128 * i: 128 * (i + 1), 128 * j: 128 * (j + 1)] for j in range(nkv)]
        assert uf[i] == [] and up[i] == [j for j, t in enumerate(tiles) if t.any()], i


def test_blockmask_size_ratio():
    """Paper review sec. 4.1: at BS = 128 the BlockMask is ~16384x smaller than the
    dense mask (BS^2 index entries collapse into one)."""
    S = 4096
    bm = oracle.block_mask("and", CAUSAL, None, 1, 1, S, S)
    assert (S * S) / bm["kv_num_blocks"][0, 0].size ** 2 == 128 * 128


def test_blockmask_broadcast_batch_uses_doc_rows():
    """A DOCUMENT leaf gives one BlockMask per batch row."""
    doc = torch.stack([W.document_ids_from_lengths([128, 128]), W.document_ids_from_lengths([256])])
    bm = oracle.block_mask("and", [("causal",), ("document",)], doc, 2, 1, 256, 256)
    f0, p0 = lists(bm, b=0)
    f1, p1 = lists(bm, b=1)
    assert f0 == [[], []] and p0 == [[0], [1]]
    assert f1 == [[], [0]] and p1 == [[0], [1]]


def test_blockmask_empty_kv():
    bm = oracle.block_mask("and", CAUSAL, None, 1, 1, 256, 0)
    assert bm["kv_indices"].shape == (1, 1, 2, 0)
    assert bm["kv_num_blocks"].sum() == 0 and bm["full_kv_num_blocks"].sum() == 0


# ---------------------------------------------------------------- forward pins

def _qkv(B, Hq, Hkv, S, D, seed=0, Skv=None):
    g = torch.Generator().manual_seed(seed)
    Skv = S if Skv is None else Skv
    q = torch.randn((B, Hq, S, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, Skv, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, Skv, D), generator=g).to(torch.bfloat16)
    return q, k, v


def _index_values(B, H, S, D):
    """V[kv, :] = kv (exact in bf16 for kv <= 256)."""
    assert S <= 256
    return torch.arange(S, dtype=torch.float32).view(1, 1, S, 1).expand(B, H, S, D).to(torch.bfloat16).contiguous()


def test_uniform_causal_closed_form():
    """Q = 0 makes every admitted score equal: under causal, O[q] = mean(0..q) = q/2
    for V[kv] = kv, and LSE = ln(q + 1)."""
    S, D = 200, 8
    q = torch.zeros((1, 1, S, D), dtype=torch.bfloat16)
    k = _qkv(1, 1, 1, S, D)[1]
    v = _index_values(1, 1, S, D)
    o, lse = oracle.forward(q, k, v, "and", CAUSAL, None)
    qs = np.arange(S)
    np.testing.assert_allclose(o[0, 0, :, 0], qs / 2, rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse[0, 0], np.log(qs + 1), rtol=0, atol=1e-12)


def test_uniform_sliding_closed_form():
    """causal AND (q - kv <= W) with Q = 0: O[q] = (max(0, q-W) + q) / 2."""
    S, D, Wn = 250, 4, 17
    q = torch.zeros((1, 1, S, D), dtype=torch.bfloat16)
    k = _qkv(1, 1, 1, S, D)[1]
    v = _index_values(1, 1, S, D)
    o, lse = oracle.forward(q, k, v, "and", [("causal",), ("sliding", Wn)], None)
    qs = np.arange(S)
    lo = np.maximum(0, qs - Wn)
    np.testing.assert_allclose(o[0, 0, :, 1], (lo + qs) / 2, atol=1e-10)
    np.testing.assert_allclose(lse[0, 0], np.log(qs - lo + 1), atol=1e-12)


def test_uniform_document_closed_form():
    """causal AND same-document with Q = 0: O[q] = (start of q's document + q) / 2."""
    lengths = [30, 1, 100, 69, 56]
    S, D = sum(lengths), 4
    doc = W.document_ids_from_lengths(lengths).unsqueeze(0)
    q = torch.zeros((1, 1, S, D), dtype=torch.bfloat16)
    k = _qkv(1, 1, 1, S, D)[1]
    v = _index_values(1, 1, S, D)
    o, lse = oracle.forward(q, k, v, "and", [("causal",), ("document",)], doc)
    starts = np.repeat(np.cumsum([0] + lengths[:-1]), lengths)
    qs = np.arange(S)
    np.testing.assert_allclose(o[0, 0, :, 2], (starts + qs) / 2, atol=1e-10)
    np.testing.assert_allclose(lse[0, 0], np.log(qs - starts + 1), atol=1e-12)


def test_alibi_geometric_closed_form():
    """ALiBi with Q = 0 under causal: p(kv) is proportional to r^(q-kv), r = e^-slope,
    a truncated geometric law.  With V[kv] = kv, O[q] = q - E[j] where
    E[j] = sum j r^j / sum r^j over j = 0..q; LSE = ln((1 - r^(q+1)) / (1 - r))."""
    S, D, H = 160, 4, 3
    slopes = torch.tensor([0.5, 0.125, 2.0 ** -6], dtype=torch.float32)
    q = torch.zeros((1, H, S, D), dtype=torch.bfloat16)
    k = _qkv(1, H, H, S, D)[1]
    v = _index_values(1, H, S, D)
    o, lse = oracle.forward(q, k, v, "and", CAUSAL, None, score=("alibi", slopes))
    for h in range(H):
        r = math.exp(-float(slopes[h]))
        for qi in [0, 1, 7, 100, 159]:
            j = np.arange(qi + 1)
            w = r ** j
            ej = (j * w).sum() / w.sum()
            assert o[0, h, qi, 3] == pytest.approx(qi - ej, abs=1e-9)
            assert lse[0, h, qi] == pytest.approx(math.log((1 - r ** (qi + 1)) / (1 - r)), abs=1e-12)


def test_softcap_saturates_at_cap():
    """cap * tanh(s / cap) is bounded by +-cap: one huge score (s = 16384) against
    zeros gives weight e^cap / (e^cap + n - 1); a huge negative one gives e^-cap."""
    cap, n, D = 30.0, 10, 2
    q = torch.zeros((1, 1, 2, D), dtype=torch.bfloat16)
    q[0, 0, :, 0] = bf([128.0, -128.0])
    k = torch.zeros((1, 1, n, D), dtype=torch.bfloat16)
    k[0, 0, 0, 0] = bf(128.0)                          # score 16384 (row 0) / -16384 (row 1)
    v = torch.zeros((1, 1, n, D), dtype=torch.bfloat16)
    v[0, 0, 0, 1] = bf(1.0)
    o, lse = oracle.forward(q, k, v, "and", [], None, score=("softcap", cap), scale=1.0)
    big = math.exp(cap)
    assert o[0, 0, 0, 1] == pytest.approx(big / (big + n - 1), rel=1e-14)
    assert lse[0, 0, 0] == pytest.approx(math.log(big + n - 1), rel=1e-14)
    small = math.exp(-cap)
    assert o[0, 0, 1, 1] == pytest.approx(small / (small + n - 1), rel=1e-12)


def test_softcap_small_scores_identity():
    """tanh(x) = x - x^3/3 + 2x^5/15 + O(x^7): for s = 1, cap = 30 the capped score is
    1 - 1/(3 cap^2) + 2/(15 cap^4) to ~1e-10."""
    cap, D = 30.0, 1
    q = torch.ones((1, 1, 1, D), dtype=torch.bfloat16)
    k = torch.tensor([0.0, 1.0], dtype=torch.bfloat16).view(1, 1, 2, 1)
    v = torch.tensor([0.0, 1.0], dtype=torch.bfloat16).view(1, 1, 2, 1)
    o, lse = oracle.forward(q, k, v, "and", [], None, score=("softcap", cap), scale=1.0)
    s = 1.0 - 1.0 / (3 * cap * cap) + 2.0 / (15 * cap ** 4)
    assert o[0, 0, 0, 0] == pytest.approx(math.exp(s) / (1 + math.exp(s)), abs=1e-9)


def test_bias_spike_selects_value_row():
    """A +100 bias spike at kv*(b,h,q) = (3q + 5h + b) % (q+1) (causal-admitted) makes
    O[b,h,q] = V[kv*] to double precision: pins bias indexing [b, h, q, kv]."""
    B, H, S, D = 2, 3, 64, 4
    q, k, v = _qkv(B, H, H, S, D, seed=3)
    bias = torch.zeros((B, H, S, S), dtype=torch.bfloat16)
    star = np.zeros((B, H, S), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            for qi in range(S):
                kv = (3 * qi + 5 * h + b) % (qi + 1)
                star[b, h, qi] = kv
                bias[b, h, qi, kv] = 100.0
    o, lse = oracle.forward(q, k, v, "and", CAUSAL, None, score=("bias", bias))
    vv = v.double().numpy()
    for b in range(B):
        for h in range(H):
            np.testing.assert_allclose(o[b, h], vv[b, h, star[b, h]], atol=1e-20, rtol=1e-12)


def test_bias_softcap_uniform_scores_closed_form():
    """bias then soft-cap with Q = 0: every score is 0, so the modified score is
    cap * tanh(bias / cap) and O is the softmax of those values (numpy) times V.
    Biases of N(0, 20) against cap 10 separate every other composition order."""
    B, H, S, D, cap = 1, 2, 96, 4, 10.0
    q = torch.zeros((B, H, S, D), dtype=torch.bfloat16)
    k = _qkv(B, H, H, S, D, seed=11)[1]
    v = _qkv(B, H, H, S, D, seed=12)[2]
    bias = (20 * torch.randn((B, H, S, S), generator=torch.Generator().manual_seed(13))).to(torch.bfloat16)
    o, lse = oracle.forward(q, k, v, "and", CAUSAL, None, score=("bias_softcap", bias, cap))
    bb, vv = bias.double().numpy(), v.double().numpy()
    for h in range(H):
        for qi in (0, 1, 50, 95):
            s = cap * np.tanh(bb[0, h, qi, : qi + 1] / cap)
            p = np.exp(s - s.max())
            assert lse[0, h, qi] == pytest.approx(s.max() + np.log(p.sum()), abs=1e-12)
            np.testing.assert_allclose(o[0, h, qi], (p / p.sum()) @ vv[0, h, : qi + 1], atol=1e-12)


def test_bias_softcap_reduces_to_each_mod():
    """A zero bias gives the soft-cap result; a cap far above every score gives
    the bias result (tanh(x) = x to 1e-12 for |x| < 1e-4)."""
    B, H, S, D = 1, 2, 130, 16
    q, k, v = _qkv(B, H, H, S, D, seed=14)
    zero = torch.zeros((B, H, S, S), dtype=torch.bfloat16)
    o1, l1 = oracle.forward(q, k, v, "and", CAUSAL, None, score=("bias_softcap", zero, 5.0))
    o2, l2 = oracle.forward(q, k, v, "and", CAUSAL, None, score=("softcap", 5.0))
    np.testing.assert_array_equal(o1, o2)
    bias = torch.randn((B, H, S, S), generator=torch.Generator().manual_seed(15)).to(torch.bfloat16)
    o3, l3 = oracle.forward(q, k, v, "and", CAUSAL, None, score=("bias_softcap", bias, 1e6))
    o4, l4 = oracle.forward(q, k, v, "and", CAUSAL, None, score=("bias", bias))
    np.testing.assert_allclose(o3, o4, atol=1e-9)
    np.testing.assert_allclose(l3, l4, atol=1e-9)


def test_default_scale_is_inverse_sqrt_d():
    """Scores are scaled by 1/sqrt(D) before softmax: D = 4, dot products 4 and 0
    give s = 2 and 0, so the weight of the first key is e^2 / (e^2 + 1)."""
    D = 4
    q = torch.ones((1, 1, 1, D), dtype=torch.bfloat16)
    k = torch.zeros((1, 1, 2, D), dtype=torch.bfloat16)
    k[0, 0, 0] = 1.0
    v = torch.zeros((1, 1, 2, D), dtype=torch.bfloat16)
    v[0, 0, 0] = 1.0
    o, lse = oracle.forward(q, k, v, "and", [], None)
    assert o[0, 0, 0, 0] == pytest.approx(math.exp(2) / (math.exp(2) + 1), rel=1e-14)
    assert lse[0, 0, 0] == pytest.approx(math.log(math.exp(2) + 1), rel=1e-14)


def test_scores_are_q_dot_k_not_transposed():
    """s[q, kv] = Q[q] . K[kv]: with Q rows e_0, e_1 and K rows 3 e_1, 0, row 0 sees
    scores (0, 0) and row 1 sees (3, 0)."""
    D = 2
    q = torch.tensor([[1.0, 0.0], [0.0, 1.0]]).view(1, 1, 2, D).to(torch.bfloat16)
    k = torch.tensor([[0.0, 3.0], [0.0, 0.0]]).view(1, 1, 2, D).to(torch.bfloat16)
    v = torch.tensor([[1.0, 0.0], [0.0, 0.0]]).view(1, 1, 2, D).to(torch.bfloat16)
    o, lse = oracle.forward(q, k, v, "and", [], None, scale=1.0)
    assert o[0, 0, 0, 0] == pytest.approx(0.5, rel=1e-15)
    assert o[0, 0, 1, 0] == pytest.approx(math.exp(3) / (math.exp(3) + 1), rel=1e-14)


def test_gqa_head_map():
    """Hq = 4, Hkv = 2: query heads 0,1 read kv head 0 and heads 2,3 read kv head 1
    (consecutive groups), seen through V = 0 on head 0 and V = 1 on head 1."""
    q, k, v = _qkv(1, 4, 2, 16, 8)
    v = torch.zeros_like(v)
    v[:, 1] = 1.0
    o, lse = oracle.forward(q, k, v, "and", CAUSAL, None)
    assert np.all(o[0, :2] == 0.0)
    np.testing.assert_allclose(o[0, 2:], 1.0, atol=1e-14)


def _sdpa_reference(q, k, v, mask, scale):
    G = q.shape[1] // k.shape[1]
    kk = k.double().repeat_interleave(G, dim=1)
    vv = v.double().repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q.double(), kk, vv, attn_mask=mask, scale=scale)


@pytest.mark.parametrize("kind,op,leaves,kw", DENSE_CASES, ids=[c[0] for c in DENSE_CASES])
def test_forward_matches_library_sdpa(kind, op, leaves, kw):
    """No score_mod + boolean mask reduces to textbook attention; cross-check with
    torch's fp64 scaled_dot_product_attention (GQA by repeating kv heads)."""
    S, D = 300, 32
    q, k, v = _qkv(2, 4, 2, S, D, seed=11)
    doc = None
    if "lengths" in kw:
        doc = W.document_ids_from_lengths(kw["lengths"]).unsqueeze(0)
        kw = dict(kw, lengths=kw["lengths"])
    dense = _torch_dense(kind, S, S, **kw)
    o, lse = oracle.forward(q, k, v, op, leaves, doc)
    ref = _sdpa_reference(q, k, v, dense, 1.0 / math.sqrt(D)).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)


def test_forward_alibi_matches_additive_sdpa():
    """ALiBi as an additive float mask slope[h] * (kv - q), plus -inf above the diagonal."""
    S, D, H = 200, 16, 4
    q, k, v = _qkv(1, H, H, S, D, seed=5)
    slopes = W.alibi_slopes(H)
    o, lse = oracle.forward(q, k, v, "and", CAUSAL, None, score=("alibi", slopes))
    idx = torch.arange(S, dtype=torch.float64)
    rel = idx.view(1, S) - idx.view(S, 1)
    add = slopes.double().view(H, 1, 1) * rel.view(1, S, S)
    add = add.masked_fill(~torch.tril(torch.ones(S, S, dtype=torch.bool)), float("-inf"))
    ref = _sdpa_reference(q, k, v, add.unsqueeze(0), 1.0 / math.sqrt(D)).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)


def test_forward_bias_and_lse_match_library():
    """Bias as an additive mask; LSE equals torch.logsumexp of the modified scores."""
    S, D, H = 150, 16, 2
    q, k, v = _qkv(1, H, H, S, D, seed=6)
    bias = torch.randn((1, H, S, S), generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    o, lse = oracle.forward(q, k, v, "and", CAUSAL, None, score=("bias", bias))
    keep = torch.tril(torch.ones(S, S, dtype=torch.bool))
    scores = q.double() @ k.double().transpose(-1, -2) / math.sqrt(D) + bias.double()
    scores = scores.masked_fill(~keep, float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(scores, dim=-1).numpy(), atol=1e-12)
    ref = _sdpa_reference(q, k, v, bias.double().masked_fill(~keep, float("-inf")), 1.0 / math.sqrt(D)).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)


# ---------------------------------------------------------------- invariants

def test_rows_sum_to_one_and_masked_are_zero():
    w = W.config(0)
    q, k, v = W.qkv(w)
    for (b, h, qi) in [(0, 0, 0), (0, 1, 77), (0, 0, 255)]:
        p, lse = oracle.prob_row(q, k, v, "and", CAUSAL, None, b, h, qi)
        assert abs(p.sum() - 1.0) < 1e-12
        assert np.all(p[qi + 1:] == 0.0) and np.all(p[: qi + 1] > 0.0)


def test_mask_as_score_identity_is_bitwise():
    """attention-gym "Concepts": any mask_mod is a score_mod returning -inf for masked
    positions.  Causal mask vs an all-attend mask plus a 0 / -inf bias: identical bits."""
    S, D, H = 192, 32, 2
    q, k, v = _qkv(1, H, H, S, D, seed=8)
    o1, l1 = oracle.forward(q, k, v, "and", CAUSAL, None)
    keep = torch.tril(torch.ones(S, S, dtype=torch.bool))
    bias = torch.zeros((1, H, S, S), dtype=torch.bfloat16).masked_fill(~keep, float("-inf"))
    o2, l2 = oracle.forward(q, k, v, "and", [], None, score=("bias", bias))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_value_ones_gives_ones():
    S, D, H = 100, 8, 2
    q, k, v = _qkv(1, H, H, S, D, seed=2)
    v = torch.ones_like(v)
    o, lse = oracle.forward(q, k, v, "and", [("causal",), ("sliding", 10)], None, score=("alibi", W.alibi_slopes(H)))
    np.testing.assert_allclose(o, 1.0, atol=1e-14)


def test_masked_keys_do_not_matter():
    """Under causal, rows q < 128 never see K/V at kv >= 128: perturbing those keys
    and values leaves their outputs bit-identical."""
    S, D = 256, 16
    q, k, v = _qkv(1, 1, 1, S, D, seed=4)
    o1, l1 = oracle.forward(q, k, v, "and", CAUSAL, None, score=("alibi", torch.tensor([0.25])))
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 128:] = 7.0
    v2[:, :, 128:] = -3.0
    o2, l2 = oracle.forward(q, k2, v2, "and", CAUSAL, None, score=("alibi", torch.tensor([0.25])))
    assert np.array_equal(o1[:, :, :128], o2[:, :, :128]) and np.array_equal(l1[:, :, :128], l2[:, :, :128])
    assert not np.array_equal(o1[:, :, 128:], o2[:, :, 128:])


def test_fully_masked_rows_and_empty_kv():
    """A row with no admitted key gives O = 0 and LSE = -inf; so does kv_len = 0."""
    q, k, v = _qkv(1, 1, 1, 20, 8)
    o, lse = oracle.forward(q, k, v, "and", [("causal",), ("sliding", -1)], None)
    assert np.all(o == 0.0) and np.all(np.isneginf(lse))
    k0, v0 = k[:, :, :0], v[:, :, :0]
    o, lse = oracle.forward(q, k0, v0, "and", CAUSAL, None)
    assert np.all(o == 0.0) and np.all(np.isneginf(lse))


def test_sampled_rows_equal_full_run():
    w = W.config(0)
    q, k, v = W.qkv(w)
    o, lse = oracle.forward(q, k, v, "and", CAUSAL, None)
    rows = W.random_rows(w, 50)
    os_, ls_ = oracle.forward(q, k, v, "and", CAUSAL, None, rows=rows)
    r = rows.numpy()
    assert np.array_equal(os_, o[r[:, 0], r[:, 1], r[:, 2]])
    assert np.array_equal(ls_, lse[r[:, 0], r[:, 1], r[:, 2]])


# ---------------------------------------------------------------- paged KV cache

def _paged(k, seed, extra=3):
    """k [B, Hkv, S, D] scattered into pages [P, Hkv, 128, D] by a seeded
    permutation (plus unused pages of noise); returns pages and the page table."""
    B, H, S, D = k.shape
    nkv = -(-S // 128)
    g = torch.Generator().manual_seed(seed)
    P = B * nkv + extra
    pages = torch.randn((P, H, 128, D), generator=g).to(torch.bfloat16)
    perm = torch.randperm(P, generator=g)[: B * nkv].view(B, nkv)
    for b in range(B):
        for kb in range(nkv):
            n = min(128, S - 128 * kb)
            pages[perm[b, kb], :, :n] = k[b, :, 128 * kb: 128 * kb + n]
    return pages, perm.to(torch.int32)


def test_paged_forward_equals_contiguous_forward():
    """Paper review sec. 4.5 (kv indices as a page table): attention over a paged
    cache equals attention over the logical K, V it maps, bit for bit."""
    B, Hq, Hkv, S, D = 2, 4, 2, 300, 16
    q, k, v = _qkv(B, Hq, Hkv, S, D, seed=40)
    kp, pt = _paged(k, 41)
    vp = torch.zeros_like(kp)
    vp_pages, _ = _paged(v, 41)  # same seed: same page permutation
    o1, l1 = oracle.forward(q, k, v, "and", CAUSAL, None)
    o2, l2 = oracle.forward_paged(q, kp, vp_pages, pt, S, "and", CAUSAL, None)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_paged_gather_shared_prefix_pages():
    """Two sequences sharing their first page (a common prefix) read the same
    physical keys: the gathered K rows coincide; with a distinct table they differ."""
    pages = torch.randn((4, 1, 128, 8), generator=torch.Generator().manual_seed(42)).to(torch.bfloat16)
    pt = torch.tensor([[2, 0], [2, 3]], dtype=torch.int32)
    k = oracle.gather_pages(pages, pt, 200)
    assert torch.equal(k[0, :, :128], k[1, :, :128]) and torch.equal(k[0, :, :128], pages[2])
    assert torch.equal(k[1, :, 128:200], pages[3, :, :72]) and not torch.equal(k[0, :, 128:], k[1, :, 128:])


# ---------------------------------------------------------------- query offset (decoding)

@pytest.mark.parametrize("op,leaves,score", [
    ("and", CAUSAL, ("none",)),
    ("and", [("causal",), ("sliding", 70)], ("alibi",)),
    ("and", [("causal",), ("document",)], ("bias",)),
    ("or", [("prefix", 30), ("causal",)], ("softcap", 3.0)),
])
@pytest.mark.parametrize("n", [1, 5])
def test_offset_queries_equal_the_last_rows(op, leaves, score, n):
    """Queries at positions S-n..S-1, given as n rows with q_offset = S - n (one
    decoding step, or a short continuation), get exactly the last n rows of the
    full forward pass: the masks and ALiBi see positions, not row numbers."""
    B, Hq, Hkv, S, D = 1, 4, 2, 200, 8
    q, k, v = _qkv(B, Hq, Hkv, S, D, seed=60)
    doc = W.document_ids_from_lengths([50, 90, 60]).unsqueeze(0)
    if score[0] == "alibi":
        score = ("alibi", W.alibi_slopes(Hq))
    bias = torch.randn((B, Hq, S, S), generator=torch.Generator().manual_seed(61)).to(torch.bfloat16)
    full_score = ("bias", bias) if score[0] == "bias" else score
    o, lse = oracle.forward(q, k, v, op, leaves, doc, score=full_score)
    part_score = ("bias", bias[:, :, S - n:].contiguous()) if score[0] == "bias" else score
    o2, lse2 = oracle.forward(q[:, :, S - n:].contiguous(), k, v, op, leaves, doc, score=part_score, q_offset=S - n)
    np.testing.assert_array_equal(o2, o[:, :, S - n:])
    np.testing.assert_array_equal(lse2, lse[:, :, S - n:])


def test_offset_block_mask_is_a_row_slice():
    """The BlockMask of 128 queries at offset 128 j is query block j of the full one."""
    S = 640
    full = oracle.block_mask("and", [("causal",), ("sliding", 200)], None, 1, 1, S, S)
    for j in range(5):
        part = oracle.block_mask("and", [("causal",), ("sliding", 200)], None, 1, 1, 128, S, q_offset=128 * j)
        for key in full:
            np.testing.assert_array_equal(part[key][0, 0, 0], full[key][0, 0, j])

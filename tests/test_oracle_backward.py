"""Pins for the oracle's backward pass (dQ, dK, dV given dO) and its transposed
BlockMask, without a GPU: torch fp64 autograd through scaled_dot_product_attention
(a library routine, GQA by repeating kv heads), central differences of the pinned
forward pass on bf16-representable steps, and invariants of the softmax gradient.
A dropped term (the row term of dS, the score_mod derivative, the scale), a
transposed operand or a wrong GQA reduction fails at least one of them."""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

CAUSAL = [("causal",)]


def _inputs(B, Hq, Hkv, Sq, D, seed, Skv=None, int_valued=False):
    g = torch.Generator().manual_seed(seed)
    Skv = Sq if Skv is None else Skv
    mk = (lambda s: torch.randint(-3, 4, s, generator=g).float()) if int_valued else (lambda s: torch.randn(s, generator=g))
    q = mk((B, Hq, Sq, D)).to(torch.bfloat16)
    k = mk((B, Hkv, Skv, D)).to(torch.bfloat16)
    v = mk((B, Hkv, Skv, D)).to(torch.bfloat16)
    do = torch.randn((B, Hq, Sq, D), generator=g).to(torch.bfloat16)
    return q, k, v, do


def _autograd(q, k, v, do, mask, scale):
    """torch fp64 SDPA and its autograd gradients; kv heads repeated for GQA, so
    their gradients are summed over the group by autograd."""
    G = q.shape[1] // k.shape[1]
    qq = q.double().requires_grad_()
    kk = k.double().requires_grad_()
    vv = v.double().requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(
        qq, kk.repeat_interleave(G, dim=1), vv.repeat_interleave(G, dim=1), attn_mask=mask, scale=scale)
    o.backward(do.double())
    return qq.grad.numpy(), kk.grad.numpy(), vv.grad.numpy()


def _dense(kind, Sq, Skv, **kw):
    ones = torch.ones((Sq, Skv), dtype=torch.bool)
    if kind == "causal":
        return torch.tril(ones)
    if kind == "sliding":
        return torch.tril(ones) & torch.triu(ones, diagonal=-kw["W"])
    if kind == "document":
        return torch.tril(ones) & torch.block_diag(*[torch.ones((n, n), dtype=torch.bool) for n in kw["lengths"]])
    if kind == "prefix_or_causal":
        m = torch.tril(ones).clone()
        m[:, : kw["P"]] = True
        return m
    if kind == "none":
        return ones
    raise KeyError(kind)


CASES = [
    ("causal", "and", CAUSAL, {}),
    ("sliding", "and", [("causal",), ("sliding", 29)], {"W": 29}),
    ("document", "and", [("causal",), ("document",)], {"lengths": [40, 3, 100, 57]}),
    ("prefix_or_causal", "or", [("prefix", 50), ("causal",)], {"P": 50}),
    ("none", "and", [], {}),
]


@pytest.mark.parametrize("kind,op,leaves,kw", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_library_autograd(kind, op, leaves, kw):
    S, D = 200, 16
    q, k, v, do = _inputs(2, 4, 2, S, D, seed=21)
    doc = W.document_ids_from_lengths(kw["lengths"]).unsqueeze(0) if "lengths" in kw else None
    dq, dk, dv = oracle.backward(q, k, v, do, op, leaves, doc)
    rq, rk, rv = _autograd(q, k, v, do, _dense(kind, S, S, **kw), 1.0 / math.sqrt(D))
    for got, want in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(got, want, atol=1e-10, rtol=0)


def test_backward_alibi_and_bias_match_additive_autograd():
    S, D, H = 150, 16, 3
    q, k, v, do = _inputs(1, H, H, S, D, seed=22)
    keep = torch.tril(torch.ones(S, S, dtype=torch.bool))
    slopes = W.alibi_slopes(H)
    idx = torch.arange(S, dtype=torch.float64)
    add = slopes.double().view(H, 1, 1) * (idx.view(1, S) - idx.view(S, 1)).view(1, S, S)
    dq, dk, dv = oracle.backward(q, k, v, do, "and", CAUSAL, None, score=("alibi", slopes))
    ref = _autograd(q, k, v, do, add.masked_fill(~keep, float("-inf")).unsqueeze(0), 1.0 / math.sqrt(D))
    for got, want in zip((dq, dk, dv), ref):
        np.testing.assert_allclose(got, want, atol=1e-10, rtol=0)
    bias = torch.randn((1, H, S, S), generator=torch.Generator().manual_seed(23)).to(torch.bfloat16)
    dq, dk, dv = oracle.backward(q, k, v, do, "and", CAUSAL, None, score=("bias", bias))
    ref = _autograd(q, k, v, do, bias.double().masked_fill(~keep, float("-inf")), 1.0 / math.sqrt(D))
    for got, want in zip((dq, dk, dv), ref):
        np.testing.assert_allclose(got, want, atol=1e-10, rtol=0)


def _loss(q, k, v, do, leaves, score):
    """sum(O * dO) from the pinned forward oracle: its gradient is the backward pass."""
    o, _ = oracle.forward(q, k, v, "and", leaves, None, score=score)
    return float((o * do.double().numpy()).sum())


@pytest.mark.parametrize("score", [("softcap", 2.0), "bias_softcap", ("none",)], ids=["softcap", "bias_softcap", "none"])
def test_backward_central_differences(score):
    """Central differences of sum(O * dO) on steps of one bf16 ulp at 1.0 (2^-7, so
    the perturbed inputs stay exact) agree with dQ, dK, dV to the O(h^2) error.
    Soft-capping has no library twin: this pins the tanh derivative."""
    B, H, S, D = 1, 2, 24, 4
    q, k, v, do = _inputs(B, H, H, S, D, seed=24)
    if score == "bias_softcap":
        score = ("bias_softcap", (2 * torch.randn((B, H, S, S), generator=torch.Generator().manual_seed(25))).to(torch.bfloat16), 1.5)
    dq, dk, dv = oracle.backward(q, k, v, do, "and", CAUSAL, None, score=score)
    h = 2.0 ** -7
    checked = 0
    for name, t, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0, 5, 1), (0, 1, 17, 3), (0, 1, 23, 0)]:
            base = t.clone()
            base[idx] = 1.0
            plus, minus = base.clone(), base.clone()
            plus[idx] = 1.0 + h
            minus[idx] = 1.0 - h
            args = {"q": q, "k": k, "v": v}
            args[name] = plus
            lp = _loss(args["q"], args["k"], args["v"], do, CAUSAL, score)
            args[name] = minus
            lm = _loss(args["q"], args["k"], args["v"], do, CAUSAL, score)
            args[name] = base
            g = oracle.backward(args["q"], args["k"], args["v"], do, "and", CAUSAL, None, score=score)
            gi = {"q": g[0], "k": g[1], "v": g[2]}[name][idx]
            fd = (lp - lm) / (2 * h)
            assert fd == pytest.approx(gi, abs=2e-3 * max(1.0, abs(gi))), (name, idx, fd, gi)
            checked += 1
    assert checked == 9


def test_dq_is_invariant_to_shifting_every_key():
    """Adding one vector c to every key row adds q.c to a whole score row, which
    softmax ignores; since each row of dS sums to 0, dQ is unchanged (integer
    inputs keep K + c exact in bf16)."""
    S, D = 96, 8
    q, k, v, do = _inputs(1, 2, 2, S, D, seed=26, int_valued=True)
    q = (q.float() / 4).to(torch.bfloat16)
    c = torch.tensor([1.0, -2.0, 0.0, 3.0, 1.0, 1.0, -1.0, 2.0]).to(torch.bfloat16)
    dq1, _, dv1 = oracle.backward(q, k, v, do, "and", CAUSAL, None, score=("alibi", W.alibi_slopes(2)))
    dq2, _, dv2 = oracle.backward(q, (k.float() + c.float()).to(torch.bfloat16), v, do, "and", CAUSAL, None,
                                  score=("alibi", W.alibi_slopes(2)))
    np.testing.assert_allclose(dq1, dq2, atol=1e-9)
    np.testing.assert_allclose(dv1, dv2, atol=1e-9)


def test_dv_column_sums_equal_do_sums():
    """Every probability row sums to 1, so sum_kv dV[kv] = sum over query rows (of
    the group's heads) of dO; rows that admit nothing contribute nothing."""
    S, D = 120, 8
    q, k, v, do = _inputs(1, 4, 2, S, D, seed=27)
    leaves = [("sliding", -1), ("prefix", 200)]  # kv >= q + 1: the last row admits nothing
    _, _, dv = oracle.backward(q, k, v, do, "and", leaves, None)
    d = do.double().numpy()
    for hk in range(2):
        want = d[0, 2 * hk: 2 * hk + 2, : S - 1].sum(axis=(0, 1))
        np.testing.assert_allclose(dv[0, hk].sum(axis=0), want, atol=1e-10)


def test_units_restrict_the_computation():
    q, k, v, do = _inputs(2, 4, 2, 64, 8, seed=28)
    full = oracle.backward(q, k, v, do, "and", CAUSAL, None)
    part = oracle.backward(q, k, v, do, "and", CAUSAL, None, units=[(1, 0)])
    np.testing.assert_array_equal(part[0][1, 0:2], full[0][1, 0:2])
    np.testing.assert_array_equal(part[1][1, 0], full[1][1, 0])
    assert np.isnan(part[0][0]).all() and np.isnan(part[2][1, 1]).all()


@pytest.mark.parametrize("leaves,kw,op", [(CAUSAL, {}, "and"), ([("causal",), ("sliding", 200)], {}, "and"),
                                          ([("prefix", 150), ("causal",)], {}, "or")])
@pytest.mark.parametrize("q_len,kv_len", [(512, 512), (300, 700), (640, 200)])
def test_transposed_block_mask_is_the_transpose(leaves, kw, op, q_len, kv_len):
    """q_* lists are the column view of kv_* lists: kb in row qb's partial (full)
    list exactly when qb is in column kb's partial (full) list, both ascending."""
    fwd = oracle.block_mask(op, leaves, None, 1, 1, q_len, kv_len)
    tr = oracle.block_mask_transposed(op, leaves, None, 1, 1, q_len, kv_len)
    nq, nkv = fwd["kv_num_blocks"].shape[2], tr["q_num_blocks"].shape[2]
    for kind, fn, fi, tn, ti in (("partial", "kv_num_blocks", "kv_indices", "q_num_blocks", "q_indices"),
                                 ("full", "full_kv_num_blocks", "full_kv_indices", "full_q_num_blocks",
                                  "full_q_indices")):
        pairs = {(qb, int(kb)) for qb in range(nq) for kb in fwd[fi][0, 0, qb, : fwd[fn][0, 0, qb]]}
        tpairs = {(int(qb), kb) for kb in range(nkv) for qb in tr[ti][0, 0, kb, : tr[tn][0, 0, kb]]}
        assert pairs == tpairs, kind
        for kb in range(nkv):
            lst = list(tr[ti][0, 0, kb, : tr[tn][0, 0, kb]])
            assert lst == sorted(lst) and all(x == 0 for x in tr[ti][0, 0, kb, tr[tn][0, 0, kb]:])


def test_transposed_causal_closed_form():
    """Causal at S = 128 n: kv block j is attended by query block j partially and by
    query blocks j+1..n-1 fully."""
    n = 6
    tr = oracle.block_mask_transposed("and", CAUSAL, None, 1, 1, 128 * n, 128 * n)
    for j in range(n):
        assert list(tr["q_indices"][0, 0, j, : tr["q_num_blocks"][0, 0, j]]) == [j]
        assert list(tr["full_q_indices"][0, 0, j, : tr["full_q_num_blocks"][0, 0, j]]) == list(range(j + 1, n))


def test_offset_backward_equals_last_rows():
    """Gradients of n query rows at offset S - n: their dQ rows equal the last dQ
    rows of the full problem whose other rows have dO = 0 (those rows then
    contribute nothing to dK and dV either)."""
    B, H, S, D, n = 1, 2, 150, 8, 20
    q, k, v, do = _inputs(B, H, H, S, D, seed=35)
    do = do.clone()
    do[:, :, : S - n] = 0
    leaves = [("causal",), ("sliding", 60)]
    score = ("alibi", W.alibi_slopes(H))
    fq, fk, fv = oracle.backward(q, k, v, do, "and", leaves, None, score=score)
    oq, ok, ov = oracle.backward(q[:, :, S - n:].contiguous(), k, v, do[:, :, S - n:].contiguous(), "and", leaves,
                                 None, score=score, q_offset=S - n)
    np.testing.assert_allclose(oq, fq[:, :, S - n:], atol=1e-12)
    np.testing.assert_allclose(ok, fk, atol=1e-12)
    np.testing.assert_allclose(ov, fv, atol=1e-12)

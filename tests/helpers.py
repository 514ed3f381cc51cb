"""Shared test helpers: tolerances and workload plumbing (no attention arithmetic)."""

import numpy as np
import torch

import workloads as W

# Tolerances against the fp64 oracle for bf16 inputs: O within 2e-2 max-abs and
# 1e-2 max-rel (norm-wise: max |O - ref| / max |ref|); LSE within 1e-3 (natural
# log).  BlockMask tensors bit-exact.
O_ABS = 2e-2
O_REL = 1e-2
LSE_ABS = 1e-3


def assert_forward_close(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    o = o_gpu.float().cpu().numpy() if torch.is_tensor(o_gpu) else np.asarray(o_gpu, dtype=np.float64)
    lse = lse_gpu.float().cpu().numpy() if torch.is_tensor(lse_gpu) else np.asarray(lse_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref)
    lse_ref = np.asarray(lse_ref)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite O"
    err = np.abs(o - o_ref).max() if o.size else 0.0
    scale = np.abs(o_ref).max() if o.size else 1.0
    assert err <= O_ABS, f"{what}: max|O-ref| = {err:.3e}"
    if scale > 0:
        assert err / scale <= O_REL, f"{what}: max|O-ref|/max|ref| = {err / scale:.3e}"
    neg = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), neg), f"{what}: -inf LSE pattern differs"
    if (~neg).any():
        lerr = np.abs(lse[~neg] - lse_ref[~neg]).max()
        assert lerr <= LSE_ABS, f"{what}: max|LSE-ref| = {lerr:.3e}"
    return err


def block_mask_equal(gpu: dict, ref: dict):
    for key in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices"):
        a, b = np.asarray(gpu[key]), np.asarray(ref[key])
        assert a.shape == b.shape, (key, a.shape, b.shape)
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)[:5]
            raise AssertionError(f"{key} differs at {bad.tolist()}")


def workload_inputs(w: W.Workload):
    """CPU inputs of a workload: q, k, v, doc_ids (or None), score spec for the oracle."""
    q, k, v = W.qkv(w)
    doc = W.document_ids(w)
    if w.score == "alibi":
        score = ("alibi", W.alibi_slopes(w.Hq))
    elif w.score == "softcap":
        score = ("softcap", w.softcap)
    elif w.score == "bias":
        score = ("bias", W.bias(w, 0))
    else:
        score = ("none",)
    return q, k, v, doc, score


def gpu_score(score, device="cuda"):
    if score[0] == "none":
        return None
    if score[0] in ("alibi", "bias", "bias_softcap"):
        return (score[0], score[1].to(device)) + tuple(score[2:])
    return score


def block_mask_extents(w: W.Workload):
    """BlockMask (B, H): one row per batch only when a document leaf is present."""
    return (w.B if w.has_document else 1), 1

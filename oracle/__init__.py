"""ctypes wrapper around the fp64 CPU oracle (``flex_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The tests, the package smoke check and the benchmark's
CPU-baseline leg are the only callers.  The CUDA library never imports this module
and this module never imports the CUDA library; the two share only the seeded
input generators in ``workloads``.

Every function follows one definition on the FlexAttention pages, cited in
``flex_oracle.c``: the mask predicates (attention-gym "Concepts", sections
"mask_mod" and "Composing masks"; paper review sec. 4.4 and 5.3), the score mods
("score_mod" section; paper review sec. 2.1; attention-gym issue "Dynamic Bias
Tensor"), block classification ("BlockMask Internals") and the attention formula
(paper review sec. 2.1).

Mask specs are ``(op, leaves, doc_ids)`` with op in {"and", "or"}, leaves a
sequence of ``("causal",)``, ``("sliding", W)``, ``("document",)`` or
``("prefix", P)``, and doc_ids an int32 tensor [B', L] (or None).  Score specs are
``("none",)``, ``("alibi", slopes[Hq] fp32)``, ``("softcap", cap)``,
``("bias", bias[B, Hq, Sq, Skv] bf16)`` or ``("bias_softcap", bias, cap)`` (the
bias added first, then the sum capped).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flex_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libflexoracle.so")

LEAF = {"causal": 0, "sliding": 1, "document": 2, "prefix": 3}
OP = {"and": 0, "or": 1}
SCORE = {"none": 0, "alibi": 1, "softcap": 2, "bias": 3, "bias_softcap": 4}
EMPTY, PARTIAL, FULL = 0, 1, 2
MAX_LEAVES = 4


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into oracle/_build/libflexoracle.so."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Mask(ctypes.Structure):
    _fields_ = [("n_leaves", ctypes.c_int32), ("op", ctypes.c_int32),
                ("kind", ctypes.c_int32 * MAX_LEAVES), ("param", ctypes.c_int64 * MAX_LEAVES),
                ("doc_ids", ctypes.c_void_p), ("doc_len", ctypes.c_int64),
                ("doc_B", ctypes.c_int32), ("pad_", ctypes.c_int32), ("q_offset", ctypes.c_int64)]


class _Problem(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("q_stride", ctypes.c_int64 * 4),
                ("k", ctypes.c_void_p), ("k_stride", ctypes.c_int64 * 4),
                ("v", ctypes.c_void_p), ("v_stride", ctypes.c_int64 * 4),
                ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
                ("q_len", ctypes.c_int64), ("kv_len", ctypes.c_int64),
                ("scale", ctypes.c_double), ("score_kind", ctypes.c_int32), ("pad_", ctypes.c_int32),
                ("slopes", ctypes.c_void_p), ("softcap", ctypes.c_double),
                ("bias", ctypes.c_void_p), ("bias_stride", ctypes.c_int64 * 4), ("q_offset", ctypes.c_int64)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, M = ctypes.POINTER(_Problem), ctypes.POINTER(_Mask)
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        lib.orc_mask_value.argtypes = [M, ctypes.c_int, ctypes.c_int, i64, i64]
        lib.orc_dense_mask.argtypes = [M, ctypes.c_int, ctypes.c_int, i64, i64, vp]
        lib.orc_block_class.argtypes = [M, ctypes.c_int, ctypes.c_int, i64, i64, ctypes.c_int, i64, i64]
        lib.orc_block_mask.argtypes = [M, ctypes.c_int, ctypes.c_int, i64, i64, ctypes.c_int,
                                       vp, vp, vp, vp, ctypes.c_int, ctypes.c_int]
        lib.orc_prob_row.argtypes = [P, M, ctypes.c_int, ctypes.c_int, i64, vp]
        lib.orc_prob_row.restype = ctypes.c_double
        lib.orc_forward_rows.argtypes = [P, M, vp, i64, vp, vp, ctypes.c_int]
        lib.orc_backward.argtypes = [P, M, vp, vp, vp, i64, vp, vp, vp, ctypes.c_int]
        lib.orc_block_mask_transposed.argtypes = [M, ctypes.c_int, ctypes.c_int, i64, i64, ctypes.c_int,
                                                  vp, vp, vp, vp]
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _mask_struct(op: str, leaves: Sequence[tuple], doc_ids: Optional[torch.Tensor], q_offset: int = 0):
    if len(leaves) > MAX_LEAVES:
        raise ValueError("at most 4 mask leaves")
    m = _Mask()
    m.q_offset = int(q_offset)
    m.n_leaves = len(leaves)
    m.op = OP[op]
    keep = []
    for i, leaf in enumerate(leaves):
        m.kind[i] = LEAF[leaf[0]]
        m.param[i] = int(leaf[1]) if len(leaf) > 1 else 0
        if leaf[0] == "document" and doc_ids is None:
            raise ValueError("document leaf needs doc_ids")
    if doc_ids is not None:
        d = doc_ids.to(torch.int32).contiguous()
        if d.dim() == 1:
            d = d.unsqueeze(0)
        keep.append(d)
        m.doc_ids = d.data_ptr()
        m.doc_B = d.shape[0]
        m.doc_len = d.shape[1]
    else:
        m.doc_B = 1
    return m, keep


def mask_value(op, leaves, doc_ids, b, h, q, kv) -> bool:
    m, keep = _mask_struct(op, leaves, doc_ids)
    return bool(_load().orc_mask_value(ctypes.byref(m), b, h, q, kv))


def dense_mask(op, leaves, doc_ids, b: int, h: int, q_len: int, kv_len: int) -> np.ndarray:
    """The materialised boolean mask [q_len, kv_len] of one (b, h)."""
    m, keep = _mask_struct(op, leaves, doc_ids)
    out = np.zeros((q_len, kv_len), dtype=np.uint8)
    _load().orc_dense_mask(ctypes.byref(m), b, h, q_len, kv_len, out.ctypes.data)
    return out.astype(bool)


def block_class(op, leaves, doc_ids, b, h, q_len, kv_len, qb, kb, block_size: int = 128) -> int:
    m, keep = _mask_struct(op, leaves, doc_ids)
    return int(_load().orc_block_class(ctypes.byref(m), b, h, q_len, kv_len, block_size, qb, kb))


def block_mask(op, leaves, doc_ids, B: int, H: int, q_len: int, kv_len: int,
               block_size: int = 128, n_threads: Optional[int] = None, split_full: bool = True,
               q_offset: int = 0) -> dict:
    """create_block_mask: dict of int32 arrays kv_num_blocks [B,H,nq], kv_indices
    [B,H,nq,nkv], full_kv_num_blocks, full_kv_indices.  split_full=False: no
    full / partial split, every non-empty block in kv_indices.  Query row i sits
    at position q_offset + i."""
    m, keep = _mask_struct(op, leaves, doc_ids, q_offset)
    nq = (q_len + block_size - 1) // block_size
    nkv = (kv_len + block_size - 1) // block_size
    kv_num = np.zeros((B, H, nq), dtype=np.int32)
    full_num = np.zeros((B, H, nq), dtype=np.int32)
    kv_idx = np.zeros((B, H, nq, nkv), dtype=np.int32)
    full_idx = np.zeros((B, H, nq, nkv), dtype=np.int32)
    rc = _load().orc_block_mask(ctypes.byref(m), B, H, q_len, kv_len, block_size,
                                kv_num.ctypes.data, kv_idx.ctypes.data,
                                full_num.ctypes.data, full_idx.ctypes.data,
                                n_threads or default_threads(), 1 if split_full else 0)
    if rc != 0:
        raise ValueError("bad block size")
    return {"kv_num_blocks": kv_num, "kv_indices": kv_idx,
            "full_kv_num_blocks": full_num, "full_kv_indices": full_idx}


def block_mask_transposed(op, leaves, doc_ids, B: int, H: int, q_len: int, kv_len: int,
                          block_size: int = 128) -> dict:
    """The transposed BlockMask: q_num_blocks [B,H,nkv], q_indices [B,H,nkv,nq]
    (partial tiles) and full_q_num_blocks / full_q_indices (full tiles)."""
    m, keep = _mask_struct(op, leaves, doc_ids)
    nq = (q_len + block_size - 1) // block_size
    nkv = (kv_len + block_size - 1) // block_size
    q_num = np.zeros((B, H, nkv), dtype=np.int32)
    full_num = np.zeros((B, H, nkv), dtype=np.int32)
    q_idx = np.zeros((B, H, nkv, nq), dtype=np.int32)
    full_idx = np.zeros((B, H, nkv, nq), dtype=np.int32)
    rc = _load().orc_block_mask_transposed(ctypes.byref(m), B, H, q_len, kv_len, block_size,
                                           q_num.ctypes.data, q_idx.ctypes.data,
                                           full_num.ctypes.data, full_idx.ctypes.data)
    if rc != 0:
        raise ValueError("bad block size")
    return {"q_num_blocks": q_num, "q_indices": q_idx, "full_q_num_blocks": full_num, "full_q_indices": full_idx}


def _bf16_view(t: torch.Tensor):
    if t.dtype != torch.bfloat16 or t.device.type != "cpu":
        raise TypeError("oracle inputs are CPU bf16 tensors")
    return t.data_ptr(), list(t.stride())


def _problem(q, k, v, score, scale, q_offset=0):
    p = _Problem()
    p.q_offset = int(q_offset)
    keep = [q, k, v]
    p.q, qs = _bf16_view(q)
    p.k, ks = _bf16_view(k)
    p.v, vs = _bf16_view(v)
    for i in range(4):
        p.q_stride[i], p.k_stride[i], p.v_stride[i] = qs[i], ks[i], vs[i]
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    p.B, p.Hq, p.Hkv, p.D = B, Hq, Hkv, D
    p.q_len, p.kv_len = Sq, Skv
    p.scale = float(scale) if scale is not None else 1.0 / (D ** 0.5)
    kind = score[0]
    p.score_kind = SCORE[kind]
    if kind == "alibi":
        sl = score[1].to(torch.float32).contiguous()
        keep.append(sl)
        p.slopes = sl.data_ptr()
    elif kind == "softcap":
        p.softcap = float(score[1])
    elif kind in ("bias", "bias_softcap"):
        bt = score[1]
        keep.append(bt)
        p.bias, bst = _bf16_view(bt)
        for i in range(4):
            p.bias_stride[i] = bst[i]
        if kind == "bias_softcap":
            p.softcap = float(score[2])
    return p, keep


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, op: str, leaves, doc_ids,
            score: tuple = ("none",), scale: Optional[float] = None,
            rows: Optional[torch.Tensor] = None, n_threads: Optional[int] = None, q_offset: int = 0):
    """The forward pass in fp64.

    With rows=None: returns O [B,Hq,Sq,D] and LSE [B,Hq,Sq] (float64 numpy).
    With rows an int64 [n,3] of (b, hq, q): returns O [n,D] and LSE [n].
    q_offset: position of query row 0 in the sequence (masks and ALiBi see
    q_offset + row; decoding steps after a cache of q_offset keys).
    """
    p, keep = _problem(q, k, v, score, scale, q_offset)
    m, keep2 = _mask_struct(op, leaves, doc_ids, q_offset)
    B, Hq, Sq, D = q.shape
    full = rows is None
    if full:
        bb, hh, qq = torch.meshgrid(torch.arange(B), torch.arange(Hq), torch.arange(Sq), indexing="ij")
        rows = torch.stack([bb.reshape(-1), hh.reshape(-1), qq.reshape(-1)], dim=1)
    r = rows.to(torch.int64).contiguous()
    n = r.shape[0]
    o = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = _load().orc_forward_rows(ctypes.byref(p), ctypes.byref(m), r.data_ptr(), n,
                                  o.ctypes.data, lse.ctypes.data, n_threads or default_threads())
    if rc != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    if full:
        return o.reshape(B, Hq, Sq, D), lse.reshape(B, Hq, Sq)
    return o, lse


def gather_pages(pages: torch.Tensor, page_table: torch.Tensor, kv_len: int) -> torch.Tensor:
    """The logical K (or V) [B, Hkv, kv_len, D] of a paged cache: logical kv block
    kb of batch b is physical page page_table[b, kb] of pages [P, Hkv, 128, D]
    (paper review sec. 4.5: the BlockMask's kv indices used as a page table)."""
    nkv = (kv_len + 127) // 128
    B = page_table.shape[0]
    idx = page_table[:, :nkv].to(torch.int64)                      # [B, nkv]
    g = pages[idx.reshape(-1)]                                      # [B*nkv, Hkv, 128, D]
    g = g.reshape(B, nkv, pages.shape[1], 128, pages.shape[3]).permute(0, 2, 1, 3, 4)
    return g.reshape(B, pages.shape[1], nkv * 128, pages.shape[3])[:, :, :kv_len].contiguous()


def forward_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, page_table: torch.Tensor,
                  kv_len: int, op: str, leaves, doc_ids, score: tuple = ("none",), scale: Optional[float] = None,
                  rows: Optional[torch.Tensor] = None, n_threads: Optional[int] = None):
    """The forward pass over a paged KV cache: the plain forward pass on the
    gathered logical K and V."""
    k = gather_pages(k_pages, page_table, kv_len)
    v = gather_pages(v_pages, page_table, kv_len)
    return forward(q, k, v, op, leaves, doc_ids, score=score, scale=scale, rows=rows, n_threads=n_threads)


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, do: torch.Tensor, op: str, leaves, doc_ids,
             score: tuple = ("none",), scale: Optional[float] = None, units=None,
             n_threads: Optional[int] = None, q_offset: int = 0):
    """Gradients of the forward pass in fp64 for upstream gradient dO (bf16 like Q).

    Returns dQ [B,Hq,Sq,D], dK and dV [B,Hkv,Skv,D] (float64 numpy).  With units a
    list of (b, hkv) pairs only those kv heads (and the query heads that read
    them) are computed; the other entries are NaN."""
    p, keep = _problem(q, k, v, score, scale, q_offset)
    m, keep2 = _mask_struct(op, leaves, doc_ids, q_offset)
    dptr, dst = _bf16_view(do)
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    if units is None:
        units = [(b, h) for b in range(B) for h in range(Hkv)]
    u = np.ascontiguousarray(np.asarray(units, dtype=np.int32).reshape(-1, 2))
    st = (ctypes.c_int64 * 4)(*dst)
    dq = np.full((B, Hq, Sq, D), np.nan)
    dk = np.full((B, Hkv, Skv, D), np.nan)
    dv = np.full((B, Hkv, Skv, D), np.nan)
    rc = _load().orc_backward(ctypes.byref(p), ctypes.byref(m), dptr, st, u.ctypes.data, u.shape[0],
                              dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, n_threads or default_threads())
    if rc != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return dq, dk, dv


def prob_row(q, k, v, op, leaves, doc_ids, b, h, qi, score=("none",), scale=None) -> Tuple[np.ndarray, float]:
    """The softmax probability row of one query and its LSE."""
    p, keep = _problem(q, k, v, score, scale)
    m, keep2 = _mask_struct(op, leaves, doc_ids)
    out = np.zeros((k.shape[2],), dtype=np.float64)
    lse = _load().orc_prob_row(ctypes.byref(p), ctypes.byref(m), b, h, qi, out.ctypes.data)
    return out, float(lse)


def workload_mask(w) -> tuple:
    """(op, leaves) of a workloads.Workload, for convenience."""
    return w.mask_op, list(w.mask_leaves)

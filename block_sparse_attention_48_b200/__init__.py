"""Python binding of the B200 block-sparse FlexAttention library (libflexattn.so).

Argument marshalling only: every step of the computation runs in the CUDA kernels
behind the C ABI of ``include/flexattn.h``.  PyTorch provides device memory and
streams.  There is no CPU fallback: importing this module without the built
library raises.

    bm = create_block_mask("and", [("causal",)], B=1, H=1, q_len=S, kv_len=S)
    o, lse = flex_attention(q, k, v, bm, score_mod=("alibi", slopes))

Mask leaves: ("causal",), ("sliding", W), ("document",), ("prefix", P), combined
by "and" / "or" ("Concepts": mask_mod, Composing masks).  Score mods: None,
("alibi", slopes[Hq] fp32), ("softcap", cap), ("bias", bias[B, Hq, Sq, Skv] bf16),
("bias_softcap", bias, cap) ("Concepts": score_mod; attention-gym issue "Dynamic
Bias Tensor"; paper review sec. 2.1).
"""

from __future__ import annotations

import contextlib
import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libflexattn.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_BAD_BLOCKMASK = range(6)
BLOCK_SIZE = 128
MAX_LEAVES = 4
LEAF = {"causal": 0, "sliding": 1, "document": 2, "prefix": 3}
OP = {"and": 0, "or": 1}
SCORE = {"none": 0, "alibi": 1, "softcap": 2, "bias": 3, "bias_softcap": 4}

EXPORTS = ("fa_status_string", "fa_block_mask_shape", "fa_create_block_mask", "fa_create_block_mask_unsplit",
           "fa_workspace_size", "fa_backward_workspace_size", "fa_backward", "fa_forward_paged",
           "fa_decode_workspace_size", "fa_decode",
           "fa_forward", "fa_get_device_status", "fa_set_watchdog_ms", "fa_set_selftest_stall",
           "fa_forward_static_scratch")


class FlexAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class MaskDesc(ctypes.Structure):
    _fields_ = [("n_leaves", ctypes.c_int32), ("op", ctypes.c_int32),
                ("kind", ctypes.c_int32 * MAX_LEAVES), ("param", ctypes.c_int64 * MAX_LEAVES),
                ("doc_ids", ctypes.c_void_p), ("doc_stride", ctypes.c_int64), ("doc_len", ctypes.c_int64),
                ("q_offset", ctypes.c_int64)]


class BlockMaskDesc(ctypes.Structure):
    _fields_ = [("kv_num_blocks", ctypes.c_void_p), ("kv_indices", ctypes.c_void_p),
                ("full_kv_num_blocks", ctypes.c_void_p), ("full_kv_indices", ctypes.c_void_p),
                ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("nq", ctypes.c_int32), ("nkv", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("has_full", ctypes.c_int32),
                ("q_len", ctypes.c_int64), ("kv_len", ctypes.c_int64), ("mask", MaskDesc),
                ("q_num_blocks", ctypes.c_void_p), ("q_indices", ctypes.c_void_p),
                ("full_q_num_blocks", ctypes.c_void_p), ("full_q_indices", ctypes.c_void_p)]


class TensorDesc(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dims", ctypes.c_int64 * 4), ("strides", ctypes.c_int64 * 4)]


class ScoreModDesc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("softcap", ctypes.c_float), ("alibi_slopes", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("bias_strides", ctypes.c_int64 * 4)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python block_sparse_attention_48_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.fa_status_string.argtypes = [ctypes.c_int]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_block_mask_shape.argtypes = [i64, i64, ctypes.c_int, ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_int32)]
    lib.fa_create_block_mask.argtypes = [ctypes.POINTER(MaskDesc), ctypes.c_int, ctypes.c_int, i64, i64,
                                         ctypes.c_int, ctypes.POINTER(BlockMaskDesc), vp]
    lib.fa_create_block_mask_unsplit.argtypes = lib.fa_create_block_mask.argtypes
    lib.fa_workspace_size.argtypes = []
    lib.fa_workspace_size.restype = ctypes.c_size_t
    lib.fa_forward.argtypes = [ctypes.POINTER(TensorDesc)] * 3 + [
        ctypes.POINTER(BlockMaskDesc), ctypes.POINTER(ScoreModDesc), ctypes.c_float,
        ctypes.POINTER(TensorDesc), vp, vp, ctypes.c_size_t, vp]
    lib.fa_backward_workspace_size.argtypes = [i64, i64, i64, i64]
    lib.fa_backward_workspace_size.restype = ctypes.c_size_t
    lib.fa_backward.argtypes = [ctypes.POINTER(TensorDesc)] * 5 + [
        vp, ctypes.POINTER(BlockMaskDesc), ctypes.POINTER(ScoreModDesc), ctypes.c_float] + \
        [ctypes.POINTER(TensorDesc)] * 3 + [vp, ctypes.c_size_t, vp]
    lib.fa_forward_paged.argtypes = [ctypes.POINTER(TensorDesc)] * 3 + [vp, i64] + [
        ctypes.POINTER(BlockMaskDesc), ctypes.POINTER(ScoreModDesc), ctypes.c_float,
        ctypes.POINTER(TensorDesc), vp, vp, ctypes.c_size_t, vp]
    lib.fa_decode_workspace_size.argtypes = [i64] * 6
    lib.fa_decode_workspace_size.restype = ctypes.c_size_t
    lib.fa_decode.argtypes = lib.fa_forward.argtypes
    lib.fa_get_device_status.argtypes = [vp, vp]
    lib.fa_set_watchdog_ms.argtypes = [ctypes.c_int]
    lib.fa_set_selftest_stall.argtypes = [ctypes.c_int]
    lib.fa_forward_static_scratch.argtypes = [ctypes.POINTER(TensorDesc)] * 3 + [
        ctypes.POINTER(BlockMaskDesc), ctypes.POINTER(ScoreModDesc), ctypes.c_float,
        ctypes.POINTER(TensorDesc), vp, vp]
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def status_string(status: int) -> str:
    return _lib.fa_status_string(int(status)).decode()


def _check(rc: int, what: str):
    if rc != FA_OK:
        raise FlexAttnError(rc, what)


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def mask_desc(op: str, leaves: Sequence[tuple], doc_ids: Optional[torch.Tensor] = None,
              q_offset: int = 0) -> MaskDesc:
    if len(leaves) > MAX_LEAVES:
        raise ValueError("at most 4 mask leaves")
    m = MaskDesc()
    m.q_offset = int(q_offset)
    m.n_leaves = len(leaves)
    m.op = OP[op]
    for i, leaf in enumerate(leaves):
        m.kind[i] = LEAF[leaf[0]]
        m.param[i] = int(leaf[1]) if len(leaf) > 1 else 0
    if doc_ids is not None:
        if doc_ids.dim() == 1:
            doc_ids = doc_ids.unsqueeze(0)
        m.doc_ids = doc_ids.data_ptr()
        m.doc_stride = doc_ids.stride(0) if doc_ids.shape[0] > 1 else 0
        m.doc_len = doc_ids.shape[1]
    return m


TRANSPOSED = ("q_num_blocks", "q_indices", "full_q_num_blocks", "full_q_indices")


class BlockMask:
    """Device BlockMask: kv_num_blocks [B,H,nq], kv_indices [B,H,nq,nkv] (partial
    blocks) and full_kv_num_blocks / full_kv_indices (full blocks), int32 on the GPU;
    with transposed=True also q_num_blocks [B,H,nkv], q_indices [B,H,nkv,nq] and the
    full_q_* pair (the view the backward pass walks)."""

    def __init__(self, desc: BlockMaskDesc, tensors: dict, keep: list):
        self.desc = desc
        self.kv_num_blocks = tensors["kv_num_blocks"]
        self.kv_indices = tensors["kv_indices"]
        self.full_kv_num_blocks = tensors["full_kv_num_blocks"]
        self.full_kv_indices = tensors["full_kv_indices"]
        self.transposed = {k: tensors[k] for k in TRANSPOSED if k in tensors}
        self._keep = keep

    @property
    def shape(self) -> Tuple[int, int, int, int]:
        return (self.desc.B, self.desc.H, self.desc.nq, self.desc.nkv)

    def to_cpu(self) -> dict:
        return {"kv_num_blocks": self.kv_num_blocks.cpu().numpy(), "kv_indices": self.kv_indices.cpu().numpy(),
                "full_kv_num_blocks": self.full_kv_num_blocks.cpu().numpy(),
                "full_kv_indices": self.full_kv_indices.cpu().numpy()}

    def transposed_to_cpu(self) -> dict:
        return {k: t.cpu().numpy() for k, t in self.transposed.items()}

    def sparsity(self) -> float:
        """Share of empty blocks ("Concepts", Inspecting a BlockMask)."""
        B, H, nq, nkv = self.shape
        total = B * H * nq * nkv
        if total == 0:
            return 0.0
        used = int(self.kv_num_blocks.sum().item() + self.full_kv_num_blocks.sum().item())
        return 1.0 - used / total


def create_block_mask(op: str, leaves: Sequence[tuple], B: int, H: int, q_len: int, kv_len: int,
                      doc_ids: Optional[torch.Tensor] = None, device=None,
                      stream: Optional[torch.cuda.Stream] = None, split_full: bool = True,
                      transposed: bool = False, q_offset: int = 0) -> BlockMask:
    """create_block_mask(mask_mod, B, H, Q_LEN, KV_LEN) on the GPU (fa_create_block_mask).
    split_full=False builds the BlockMask without the full / partial split
    (fa_create_block_mask_unsplit): every non-empty tile is masked per element.
    transposed=True also builds the q_* view the backward pass needs.  q_offset:
    position of query row 0 (decoding after a cache of q_offset keys)."""
    device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    nq, nkv = ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.fa_block_mask_shape(q_len, kv_len, BLOCK_SIZE, ctypes.byref(nq), ctypes.byref(nkv)),
           "fa_block_mask_shape")
    nq, nkv = nq.value, nkv.value
    keep = []
    if doc_ids is not None:
        # rows padded to a multiple of 4 ids (16 bytes): the kernels read ids in 16-byte vectors
        ids = doc_ids.to(device=device, dtype=torch.int32)
        ids = ids.unsqueeze(0) if ids.dim() == 1 else ids
        L = ids.shape[1]
        buf = torch.zeros((ids.shape[0], (L + 3) // 4 * 4), dtype=torch.int32, device=device)
        buf[:, :L] = ids
        doc_ids = buf[:, :L]
        keep.append(buf)
    t = {"kv_num_blocks": torch.empty((B, H, nq), dtype=torch.int32, device=device),
         "kv_indices": torch.empty((B, H, nq, nkv), dtype=torch.int32, device=device),
         "full_kv_num_blocks": torch.empty((B, H, nq), dtype=torch.int32, device=device),
         "full_kv_indices": torch.empty((B, H, nq, nkv), dtype=torch.int32, device=device)}
    d = BlockMaskDesc()
    d.kv_num_blocks = t["kv_num_blocks"].data_ptr()
    d.kv_indices = t["kv_indices"].data_ptr()
    d.full_kv_num_blocks = t["full_kv_num_blocks"].data_ptr()
    d.full_kv_indices = t["full_kv_indices"].data_ptr()
    if transposed:
        for name, shape in (("q_num_blocks", (B, H, nkv)), ("q_indices", (B, H, nkv, nq)),
                            ("full_q_num_blocks", (B, H, nkv)), ("full_q_indices", (B, H, nkv, nq))):
            t[name] = torch.empty(shape, dtype=torch.int32, device=device)
            setattr(d, name, t[name].data_ptr() if t[name].numel() else None)
    m = mask_desc(op, leaves, doc_ids, q_offset)
    with torch.cuda.device(device):
        fn = _lib.fa_create_block_mask if split_full else _lib.fa_create_block_mask_unsplit
        _check(fn(ctypes.byref(m), B, H, q_len, kv_len, BLOCK_SIZE, ctypes.byref(d), _stream_ptr(stream)),
               "fa_create_block_mask" if split_full else "fa_create_block_mask_unsplit")
    return BlockMask(d, t, keep)


def _expanded(t: torch.Tensor) -> bool:
    """True if a dimension of size > 1 has stride 0 (an expand()ed broadcast)."""
    return any(t.stride(i) == 0 and t.shape[i] > 1 for i in range(t.dim()))


def tensor_desc(t: torch.Tensor) -> TensorDesc:
    if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_cuda:
        raise TypeError("expected a 4-D bf16 CUDA tensor [B, H, S, D]")
    if _expanded(t):
        raise TypeError("expanded (stride-0) dimensions of size > 1 are not accepted; materialise the tensor")
    d = TensorDesc()
    d.data = t.data_ptr()
    for i in range(4):
        d.dims[i] = t.shape[i]
        d.strides[i] = t.stride(i)
    return d


_workspaces = {}


def workspace(device: torch.device) -> torch.Tensor:
    """The per-device workspace (status word) used by default; zero-filled."""
    key = device.index if device.index is not None else torch.cuda.current_device()
    ws = _workspaces.get(key)
    if ws is None:
        ws = torch.zeros((int(_lib.fa_workspace_size()),), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


_decode_workspaces = {}


def decode_workspace(device: torch.device, need: int = 0) -> torch.Tensor:
    """The per-device workspace flex_decode uses by default: zero-filled when it is
    (re)allocated, at least `need` bytes; every fa_decode call leaves it ready for
    the next.  Calls that use it run one after another (one stream)."""
    key = device.index if device.index is not None else torch.cuda.current_device()
    ws = _decode_workspaces.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros((max(need, 256),), dtype=torch.uint8, device=device)
        _decode_workspaces[key] = ws
    return ws


def score_mod_desc(score_mod) -> Tuple[ScoreModDesc, list]:
    sm = ScoreModDesc()
    keep = []
    if score_mod is None or score_mod[0] == "none":
        sm.kind = SCORE["none"]
    elif score_mod[0] == "alibi":
        slopes = score_mod[1]
        if not (slopes.is_cuda and slopes.dtype == torch.float32 and slopes.is_contiguous()):
            raise TypeError("ALiBi slopes: contiguous fp32 CUDA tensor [Hq]")
        sm.kind = SCORE["alibi"]
        sm.alibi_slopes = slopes.data_ptr()
        keep.append(slopes)
    elif score_mod[0] == "softcap":
        sm.kind = SCORE["softcap"]
        sm.softcap = float(score_mod[1])
    elif score_mod[0] in ("bias", "bias_softcap"):
        b = score_mod[1]
        if not (b.is_cuda and b.dtype == torch.bfloat16 and b.dim() == 4):
            raise TypeError("bias: bf16 CUDA tensor [B, Hq, Sq, Skv]")
        # stride 0 over batch or heads is passed through (the kernel broadcasts it)
        if b.stride(3) != 1 or any(b.stride(i) % 8 for i in range(3)) or b.data_ptr() % 16 or \
                (b.stride(2) == 0 and b.shape[2] > 1):
            # TMA needs 16-byte row strides: copy into rows padded to 8 elements
            kl = b.shape[3]
            pad = torch.zeros(b.shape[:3] + ((kl + 7) // 8 * 8,), dtype=b.dtype, device=b.device)
            pad[..., :kl] = b
            b = pad[..., :kl]
        sm.kind = SCORE[score_mod[0]]
        if score_mod[0] == "bias_softcap":
            sm.softcap = float(score_mod[2])
        sm.bias = b.data_ptr()
        for i in range(4):
            sm.bias_strides[i] = b.stride(i)
        keep.append(b)
    else:
        raise ValueError(f"unknown score_mod {score_mod[0]!r}")
    return sm, keep


def flex_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_mask: BlockMask,
                   score_mod=None, scale: Optional[float] = None, return_lse: bool = True,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   ws: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None):
    """flex_attention(q, k, v, block_mask, score_mod) -> (out, lse) through fa_forward.

    q [B,Hq,Sq,D], k/v [B,Hkv,Skv,D] bf16 CUDA tensors (D contiguous).  Returns
    out [B,Hq,Sq,D] bf16 and lse [B,Hq,Sq] fp32 (natural log), or out alone."""
    # inputs expanded over a dimension (stride 0) are materialised: the kernels
    # address tiles by coordinates
    q, k, v = (t.contiguous() if _expanded(t) else t for t in (q, k, v))
    B, Hq, Sq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, Sq, D), dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if lse is not None and not (lse.is_contiguous() and lse.dtype == torch.float32 and lse.shape == (B, Hq, Sq)):
        raise TypeError("lse: contiguous fp32 [B, Hq, Sq]")
    sm, keep = score_mod_desc(score_mod)
    ws = ws if ws is not None else workspace(q.device)
    qd, kd, vd, od = tensor_desc(q), tensor_desc(k), tensor_desc(v), tensor_desc(out)
    with torch.cuda.device(q.device):
        rc = _lib.fa_forward(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(block_mask.desc),
                             ctypes.byref(sm), ctypes.c_float(scale if scale is not None else 0.0),
                             ctypes.byref(od), ctypes.c_void_p(lse.data_ptr() if lse is not None else 0),
                             ctypes.c_void_p(ws.data_ptr()), ctypes.c_size_t(ws.numel()), _stream_ptr(stream))
    _check(rc, "fa_forward")
    return (out, lse) if return_lse else out


def flex_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_mask: BlockMask, score_mod=None,
                scale: Optional[float] = None, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """FlexDecoding (fa_decode): a few query tokens (G * q_len <= 16 per kv head)
    against a long cache, split along KV and merged.  Build the BlockMask with
    q_offset = the position of the first query token."""
    B, Hq, Sq, D = q.shape
    out = out if out is not None else torch.empty((B, Hq, Sq, D), dtype=torch.bfloat16, device=q.device)
    lse = lse if lse is not None else torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    need = int(_lib.fa_decode_workspace_size(B, Hq, k.shape[1], Sq, k.shape[2], D))
    if ws is None:
        ws = decode_workspace(q.device, need)
    elif ws.numel() < need:
        raise FlexAttnError(f"fa_decode: workspace of {ws.numel()} bytes, {need} needed")
    sm, keep = score_mod_desc(score_mod)
    qd, kd, vd, od = tensor_desc(q), tensor_desc(k), tensor_desc(v), tensor_desc(out)
    with torch.cuda.device(q.device):
        rc = _lib.fa_decode(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(block_mask.desc),
                            ctypes.byref(sm), ctypes.c_float(scale if scale is not None else 0.0), ctypes.byref(od),
                            ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                            ctypes.c_size_t(ws.numel()), _stream_ptr(stream))
    _check(rc, "fa_decode")
    return out, lse


def flex_attention_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, page_table: torch.Tensor,
                         block_mask: BlockMask, score_mod=None, scale: Optional[float] = None,
                         out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                         ws: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """flex_attention over a paged KV cache (fa_forward_paged): k_pages / v_pages
    [num_pages, Hkv, 128, D] bf16, page_table int32 [B, >= nkv] mapping logical kv
    block kb of batch b to a page; the BlockMask is over logical positions."""
    B, Hq, Sq, D = q.shape
    if not (page_table.is_cuda and page_table.dtype == torch.int32 and page_table.dim() == 2
            and page_table.stride(1) == 1):
        raise TypeError("page_table: int32 CUDA tensor [B, pages per sequence], rows contiguous")
    out = out if out is not None else torch.empty((B, Hq, Sq, D), dtype=torch.bfloat16, device=q.device)
    lse = lse if lse is not None else torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    sm, keep = score_mod_desc(score_mod)
    ws = ws if ws is not None else workspace(q.device)
    qd, kd, vd, od = tensor_desc(q), tensor_desc(k_pages), tensor_desc(v_pages), tensor_desc(out)
    with torch.cuda.device(q.device):
        rc = _lib.fa_forward_paged(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd),
                                   ctypes.c_void_p(page_table.data_ptr()), page_table.stride(0),
                                   ctypes.byref(block_mask.desc), ctypes.byref(sm),
                                   ctypes.c_float(scale if scale is not None else 0.0), ctypes.byref(od),
                                   ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                   ctypes.c_size_t(ws.numel()), _stream_ptr(stream))
    _check(rc, "fa_forward_paged")
    return out, lse


def flex_attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                            lse: torch.Tensor, grad_out: torch.Tensor, block_mask: BlockMask, score_mod=None,
                            scale: Optional[float] = None, dq: Optional[torch.Tensor] = None,
                            dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
                            ws: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """Gradients (dq, dk, dv) of flex_attention through fa_backward, given the
    forward's out and lse and the upstream gradient.  block_mask must have been
    built with transposed=True.  ws, if given, is a uint8 device buffer of at least
    fa_backward_workspace_size bytes; its first word holds the device status."""
    q, k, v = (t.contiguous() if _expanded(t) else t for t in (q, k, v))
    grad_out = grad_out.contiguous() if _expanded(grad_out) else grad_out
    B, Hq, Sq, D = q.shape
    if not block_mask.transposed:
        raise ValueError("the backward pass needs a BlockMask built with transposed=True")
    if not (lse.is_contiguous() and lse.dtype == torch.float32 and lse.shape == (B, Hq, Sq)):
        raise TypeError("lse: contiguous fp32 [B, Hq, Sq]")
    dq = dq if dq is not None else torch.empty_like(q)
    dk = dk if dk is not None else torch.empty_like(k)
    dv = dv if dv is not None else torch.empty_like(v)
    need = int(_lib.fa_backward_workspace_size(B, Hq, Sq, D))
    if ws is None:
        # the prologue writes every row of the workspace it reads; only the status
        # word at its start needs a defined value
        with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
            ws = torch.empty((need,), dtype=torch.uint8, device=q.device)
            ws[:256].zero_()
    sm, keep = score_mod_desc(score_mod)
    descs = [tensor_desc(t) for t in (q, k, v, out, grad_out, dq, dk, dv)]
    with torch.cuda.device(q.device):
        rc = _lib.fa_backward(*[ctypes.byref(d) for d in descs[:5]], ctypes.c_void_p(lse.data_ptr()),
                              ctypes.byref(block_mask.desc), ctypes.byref(sm),
                              ctypes.c_float(scale if scale is not None else 0.0),
                              *[ctypes.byref(d) for d in descs[5:]], ctypes.c_void_p(ws.data_ptr()),
                              ctypes.c_size_t(ws.numel()), _stream_ptr(stream))
    _check(rc, "fa_backward")
    return dq, dk, dv


class FlexAttentionFunction(torch.autograd.Function):
    """flex_attention as a torch autograd function: forward through fa_forward,
    backward through fa_backward (the BlockMask must carry its transposed view)."""

    @staticmethod
    def forward(ctx, q, k, v, block_mask, score_mod, scale):
        out, lse = flex_attention(q, k, v, block_mask, score_mod=score_mod, scale=scale)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.block_mask, ctx.score_mod, ctx.scale = block_mask, score_mod, scale
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, grad_out, grad_lse):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = flex_attention_backward(q, k, v, out, lse, grad_out.contiguous(), ctx.block_mask,
                                             score_mod=ctx.score_mod, scale=ctx.scale)
        return dq, dk, dv, None, None, None


def flex_attention_autograd(q, k, v, block_mask: BlockMask, score_mod=None, scale: Optional[float] = None):
    """Differentiable flex_attention: returns (out, lse); out.backward() runs fa_backward."""
    return FlexAttentionFunction.apply(q, k, v, block_mask, score_mod, scale)


def device_status(ws: Optional[torch.Tensor] = None, device=None, stream=None) -> int:
    """Synchronise and return (and clear) the device status of earlier forward calls."""
    device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    ws = ws if ws is not None else workspace(device)
    return int(_lib.fa_get_device_status(ctypes.c_void_p(ws.data_ptr()), _stream_ptr(stream)))


def set_watchdog_ms(ms: int):
    _check(_lib.fa_set_watchdog_ms(int(ms)), "fa_set_watchdog_ms")


def set_selftest_stall(on: bool):
    """Watchdog self-test: while on, every forward launch stalls its producer
    until the watchdog limit runs out and reports FA_ERR_TIMEOUT."""
    _check(_lib.fa_set_selftest_stall(1 if on else 0), "fa_set_selftest_stall")

"""Seeded synthetic inputs for the block-sparse FlexAttention forward pass.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark.  It holds only input construction (shapes, seeds, random draws and the
document layout); none of the attention arithmetic lives here.

Workloads follow the attention shapes the FlexAttention pages describe: LLaMA-like
heads (D = 64 or 128), causal / sliding-window / document masks, ALiBi, tanh
soft-capping and a dynamic [B, H, S, S] bias ("Flex Attention" paper review, sec. 5.1
and 6.1; attention-gym issue "Dynamic Bias Tensor ... Without Recompilation").
There is no public dataset behind these workloads: every tensor is drawn from a
seeded generator.
"""

from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import torch

BLOCK_SIZE = 128

# Mask leaves and combining operators, by name.  The predicates themselves live in
# the oracle and in the CUDA kernels; here they are only labels.
CAUSAL = ("causal",)


def sliding(window: int) -> Tuple[str, int]:
    return ("sliding", int(window))


DOCUMENT = ("document",)
PREFIX = "prefix"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    q_len: int
    kv_len: int
    D: int
    mask_op: str                      # "and" | "or"
    mask_leaves: Tuple[tuple, ...]    # e.g. (("causal",), ("sliding", 1024))
    score: str                        # "none" | "alibi" | "softcap" | "bias"
    softcap: float = 30.0
    seed: int = 0
    doc_seed: Optional[int] = None

    @property
    def has_document(self) -> bool:
        return any(l[0] == "document" for l in self.mask_leaves)

    @property
    def scale(self) -> float:
        return 1.0 / (self.D ** 0.5)


# The five measured configurations.  Index 0 is the small case the oracle finishes
# in seconds; index 1 is the dense-causal ALiBi configuration the headline metric
# is quoted on.
CONFIGS: List[Workload] = [
    Workload("causal_b1_h2_s256_d64", 1, 2, 2, 256, 256, 64, "and", (CAUSAL,), "none", seed=0),
    Workload("causal_alibi_b4_h16_s2048_d64", 4, 16, 16, 2048, 2048, 64, "and", (CAUSAL,), "alibi", seed=1),
    Workload("swa1024_softcap30_b2_h16_s8192_d128", 2, 16, 16, 8192, 8192, 128, "and",
             (CAUSAL, sliding(1024)), "softcap", softcap=30.0, seed=2),
    Workload("doc_gqa_b1_hq32_hkv8_s16384_d128", 1, 32, 8, 16384, 16384, 128, "and",
             (CAUSAL, DOCUMENT), "none", seed=3, doc_seed=1003),
    Workload("causal_bias_b2_h8_s4096_d64", 2, 8, 8, 4096, 4096, 64, "and", (CAUSAL,), "bias", seed=4),
]


def config(i: int) -> Workload:
    return CONFIGS[i]


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def qkv(w: Workload, device: str = "cpu") -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q [B,Hq,Sq,D], K and V [B,Hkv,Skv,D] in bf16, drawn N(0,1) in fp32 in the order Q, K, V."""
    g = generator(w.seed)
    q = torch.randn((w.B, w.Hq, w.q_len, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((w.B, w.Hkv, w.kv_len, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((w.B, w.Hkv, w.kv_len, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    if device != "cpu":
        q, k, v = q.to(device), k.to(device), v.to(device)
    return q, k, v


def document_lengths(total: int, seed: int, lo: int = 256, hi: int = 4096) -> List[int]:
    """Packed document lengths drawn uniform in [lo, hi]; the last one is truncated to fit."""
    g = generator(seed)
    lengths: List[int] = []
    acc = 0
    while acc < total:
        n = int(torch.randint(lo, hi + 1, (1,), generator=g).item())
        n = min(n, total - acc)
        lengths.append(n)
        acc += n
    return lengths


def document_ids_from_lengths(lengths: Sequence[int]) -> torch.Tensor:
    """int32 ids, one per token position: position t carries the index of the document holding it."""
    ids = [torch.full((int(n),), i, dtype=torch.int32) for i, n in enumerate(lengths)]
    return torch.cat(ids) if ids else torch.zeros((0,), dtype=torch.int32)


def document_ids(w: Workload) -> Optional[torch.Tensor]:
    """[B, max(Sq, Skv)] int32 document ids (batch b drawn from seed doc_seed + b), or None."""
    if not w.has_document:
        return None
    L = max(w.q_len, w.kv_len)
    rows = []
    for b in range(w.B):
        rows.append(document_ids_from_lengths(document_lengths(L, (w.doc_seed or 0) + b)))
    return torch.stack(rows).contiguous()


def alibi_slopes(H: int) -> torch.Tensor:
    """The geometric per-head slope sequence 2^(-8(h+1)/H), fp32 (the ALiBi paper's choice)."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32)


def bias(w: Workload, call: int = 0) -> torch.Tensor:
    """Dynamic additive bias [B, Hq, Sq, Skv] bf16 ~ N(0,1); a fresh draw per call index."""
    g = generator(10_000 * (w.seed + 1) + call)
    return torch.randn((w.B, w.Hq, w.q_len, w.kv_len), generator=g, dtype=torch.float32).to(torch.bfloat16)


def random_rows(w: Workload, n: int, seed: int = 7) -> torch.Tensor:
    """n distinct seeded (b, hq, q) row triples (int64 [n,3]) for sampled checks at full size."""
    g = generator(seed)
    total = w.B * w.Hq * w.q_len
    n = min(n, total)
    flat = torch.randperm(total, generator=g)[:n]
    b = flat // (w.Hq * w.q_len)
    rem = flat % (w.Hq * w.q_len)
    h = rem // w.q_len
    q = rem % w.q_len
    return torch.stack([b, h, q], dim=1).to(torch.int64)


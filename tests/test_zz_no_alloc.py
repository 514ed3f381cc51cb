"""The allocation-free forward entry point (fa_forward_static_scratch).

It exists for callers that cannot allocate device memory when they run the
forward pass, such as an engine that plans memory up front and hands an operator
only its input and output buffers, or a serving loop that must not enter the
allocator mid-request.  Its scratch lives in a static device array instead of a
caller workspace.  Here its results, called through the C ABI, must match the
regular fa_forward entry point on the same inputs, on two calls in a row.
"""

import ctypes

import pytest
import torch

import workloads as W
from helpers import LSE_ABS, O_ABS, O_REL

pytestmark = pytest.mark.gpu


def _inputs(seed, B=1, H=2, S=300, D=64):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn((B, H, S, D), generator=g).to(torch.bfloat16).cuda() for _ in range(3)]


def test_static_scratch_forward_matches_fa_forward():
    import block_sparse_attention_48_b200 as fa

    lib = fa.library()
    S, H = 300, 2
    slopes = W.alibi_slopes(H).cuda()
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, S, S)
    stream = torch.cuda.current_stream()
    for call in range(2):
        q, k, v = _inputs(seed=40 + call)
        o_ref, lse_ref = fa.flex_attention(q, k, v, bm, score_mod=("alibi", slopes))

        o = torch.full_like(q, float("nan"))
        lse = torch.full((1, H, S), float("nan"), dtype=torch.float32, device="cuda")
        qd, kd, vd, od = (fa.tensor_desc(t) for t in (q, k, v, o))
        sm, keep = fa.score_mod_desc(("alibi", slopes))
        rc = lib.fa_forward_static_scratch(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd),
                                           ctypes.byref(bm.desc), ctypes.byref(sm), ctypes.c_float(0.0),
                                           ctypes.byref(od), ctypes.c_void_p(lse.data_ptr()),
                                           ctypes.c_void_p(stream.cuda_stream))
        assert rc == fa.FA_OK, fa.status_string(rc)
        torch.cuda.synchronize()

        err = (o.float() - o_ref.float()).abs().max().item()
        assert err <= O_ABS
        assert err / o_ref.float().abs().max().item() <= O_REL
        assert (lse - lse_ref).abs().max().item() <= LSE_ABS

#!/usr/bin/env python
"""Benchmark of the block-sparse FlexAttention forward pass on B200.

Metric: effective TFLOP/s, counting only the FLOPs of unmasked (q, kv) pairs
(4 * D per pair: QK^T and PV), for one step = build the BlockMask + run the
forward pass over one batch of synthetic inputs already resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl ours|reference]

Prints one JSON line (rank 0).  With N > 1 (launched by torch.distributed.run)
every rank runs its own full replica of the workload (independent problems, no
collective on the data path): weak scaling, value = all ranks' FLOPs / the
slowest rank's time.
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "effective TFLOP/s (unmasked FLOPs) fwd at 1 B200, % of BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------- workload arithmetic (metric definition)

def admitted_pairs(w: W.Workload, doc) -> int:
    """Number of (q, kv) pairs the workload's mask admits, over all (b, hq), from
    the closed forms of the enumerated masks used by the configurations."""
    leaves = [l[0] for l in w.mask_leaves]
    S = w.q_len
    assert w.q_len == w.kv_len and w.mask_op == "and"
    if leaves == ["causal"]:
        per_bh = S * (S + 1) // 2
        return per_bh * w.B * w.Hq
    if leaves == ["causal", "sliding"]:
        Wn = w.mask_leaves[1][1]
        per_bh = sum(min(q, Wn) + 1 for q in range(S))
        return per_bh * w.B * w.Hq
    if leaves == ["causal", "document"]:
        total = 0
        for b in range(w.B):
            ids = doc[b].tolist()
            run = 0
            for t in range(S):
                run = run + 1 if t > 0 and ids[t] == ids[t - 1] else 1
                total += run
        return total * w.Hq
    raise ValueError("no closed form for this mask")


def algorithmic_bytes(w: W.Workload, pairs: int) -> int:
    """Bytes the forward pass must move at least: Q, K, V, O (bf16), LSE (fp32) and,
    with a bias score_mod, the bias of every admitted pair (bf16)."""
    qo = 2 * w.B * w.Hq * w.q_len * w.D * 2
    kv = 2 * w.B * w.Hkv * w.kv_len * w.D * 2
    lse = w.B * w.Hq * w.q_len * 4
    bias = pairs * 2 if w.score == "bias" else 0
    return qo + kv + lse + bias


def max_over_ranks(values, world, device):
    """Element-wise maximum of per-rank timings over all ranks: in a replica run the
    slowest rank decides the job's time."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t]


def aggregate_tflops(eff_flops_per_rank, world, ms):
    """Whole-job throughput of `world` replicas: every rank's effective FLOPs over
    the slowest rank's time per step."""
    return world * eff_flops_per_rank / (ms * 1e-3) / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"]))}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=FALLBACK_PEAKS["bf16_tflops"]), "fallback"


FWD_SOURCES = ("flex_fwd_impl.cuh", "flex_fwd.cu", "flex_fwd_ext.cu", "flex_fwd_page.cu", "ptx.cuh", "mask_eval.cuh",
               "flex_fwd.cuh", "score_math.cuh", "context.cuh")
BWD_SOURCES = ("flex_bwd.cu", "flex_bwd.cuh", "ptx.cuh", "mask_eval.cuh", "flex_fwd.cuh", "score_math.cuh", "context.cuh",
               "tmap.cuh")
DEC_SOURCES = ("flex_decode.cu", "flex_decode.cuh", "decode_walk.cuh", "ptx.cuh", "mask_eval.cuh", "flex_fwd.cuh",
               "score_math.cuh", "context.cuh")
KERNEL_SOURCES = {"flex_fwd": FWD_SOURCES, "flex_bwd": BWD_SOURCES, "flex_decode": DEC_SOURCES}


def kernel_source_hash(names=FWD_SOURCES) -> str:
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "block_sparse_attention_48_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(name: str, kernel: str = "flex_fwd"):
    """DRAM bytes per launch of the forward, backward or decode kernel from the
    committed ncu summary of workload `name`, or None when absent or taken on a
    different kernel source."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{name}.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_source_hash") != kernel_source_hash(KERNEL_SOURCES[kernel]):
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        mhz, mx, reasons = [], None, set()
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(mhz)}


# ---------------------------------------------------------------- our arm

class Prepared:
    """One step through the C ABI with every ctypes argument built once.
    split_full=False builds the BlockMask without the full / partial split."""

    def __init__(self, fa, w, q, k, v, doc, score, o, lse, stream, split_full=True):
        self.fa, self.lib = fa, fa.library()
        self.stream = ctypes.c_void_p(stream.cuda_stream)
        Bm = w.B if w.has_document else 1
        self.bm = fa.create_block_mask(w.mask_op, list(w.mask_leaves), Bm, 1, w.q_len, w.kv_len, doc_ids=doc,
                                       stream=stream, split_full=split_full)
        self.build = self.lib.fa_create_block_mask if split_full else self.lib.fa_create_block_mask_unsplit
        self.Bm = Bm
        self.qd, self.kd, self.vd, self.od = (fa.tensor_desc(t) for t in (q, k, v, o))
        self.sm, self._keep = fa.score_mod_desc(score)
        self.ws = fa.workspace(q.device)
        self.lse = lse
        self.w = w

    def block_mask(self):
        w = self.w
        rc = self.build(ctypes.byref(self.bm.desc.mask), self.Bm, 1, w.q_len, w.kv_len, 128,
                        ctypes.byref(self.bm.desc), self.stream)
        if rc:
            raise RuntimeError(self.fa.status_string(rc))

    def forward(self):
        rc = self.lib.fa_forward(ctypes.byref(self.qd), ctypes.byref(self.kd), ctypes.byref(self.vd),
                                 ctypes.byref(self.bm.desc), ctypes.byref(self.sm), ctypes.c_float(0.0),
                                 ctypes.byref(self.od), ctypes.c_void_p(self.lse.data_ptr()),
                                 ctypes.c_void_p(self.ws.data_ptr()), ctypes.c_size_t(self.ws.numel()), self.stream)
        if rc:
            raise RuntimeError(self.fa.status_string(rc))


def device_score(w, score, dev):
    if score[0] in ("alibi", "bias"):
        return (score[0], score[1].to(dev))
    if score[0] == "none":
        return ("none",)
    return score


def host_score(w):
    if w.score == "alibi":
        return ("alibi", W.alibi_slopes(w.Hq))
    if w.score == "softcap":
        return ("softcap", w.softcap)
    if w.score == "bias":
        return ("bias", W.bias(w, 0))
    return ("none",)


def measure(fa, w, dev, stream, steps, warmup, world=1, split_full=True, clocks=None):
    """Time `steps` steps (BlockMask build + forward) and then `steps` forward
    launches alone, L2 flushed before each, CUDA events on the launching stream.
    Returns per-launch averages (max over ranks) and the workload's arithmetic."""
    q_h, k_h, v_h = W.qkv(w)
    doc = W.document_ids(w)
    score_h = host_score(w)
    pairs = admitted_pairs(w, doc)
    with torch.cuda.stream(stream):
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
        score = device_score(w, score_h, dev)
        biases = None
        if w.score == "bias":  # a fresh bias every call: cycle two draws, pointer and values change
            biases = [score[1], W.bias(w, 1).to(dev)]
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device=dev)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream.synchronize()
    preps = [Prepared(fa, w, q, k, v, doc, score, o, lse, stream, split_full)]
    if biases is not None:
        preps.append(Prepared(fa, w, q, k, v, doc, ("bias", biases[1]), o, lse, stream, split_full))

    for i in range(warmup):
        with torch.cuda.stream(stream):
            flush.zero_()
        preps[i % len(preps)].block_mask()
        preps[i % len(preps)].forward()
    stream.synchronize()
    status = fa.device_status(stream=stream)
    if status != 0:
        raise RuntimeError(f"device status {fa.status_string(status)} after warm-up ({w.name})")

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    ev_f = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    if clocks is not None:
        clocks.start()
        time.sleep(0.3)
    # Timed steps: events bracket the whole step only, so that the forward kernel
    # follows the BlockMask kernel directly.
    for i in range(steps):
        with torch.cuda.stream(stream):
            flush.zero_()  # L2 flush between timed steps, outside the events
        pr = preps[i % len(preps)]
        ev[i][0].record(stream)
        pr.block_mask()
        pr.forward()
        ev[i][1].record(stream)
    # The forward kernel on its own (same flushes), for its roofline.
    for i in range(steps):
        with torch.cuda.stream(stream):
            flush.zero_()
        pr = preps[i % len(preps)]
        ev_f[i][0].record(stream)
        pr.forward()
        ev_f[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop() if clocks is not None else None
    step_ms = [a.elapsed_time(b) for a, b in ev]
    fwd_ms = [a.elapsed_time(b) for a, b in ev_f]
    status = fa.device_status(stream=stream)
    if status != 0:
        raise RuntimeError(f"device status {fa.status_string(status)} after timing ({w.name})")
    ms_step, ms_fwd = max_over_ranks([sum(step_ms) / len(step_ms), sum(fwd_ms) / len(fwd_ms)], world, dev)
    del preps, q, k, v, o, lse, flush, biases, score
    return dict(ms_step=ms_step, ms_fwd=ms_fwd, eff_flops=4.0 * w.D * pairs,
                alg_bytes=algorithmic_bytes(w, pairs), pairs=pairs, clocks=clk, status="FA_OK",
                inputs=(q_h, k_h, v_h, doc, score_h))


def roofline(w, r, peaks, peak_src):
    """Roofline of the forward kernel from its CUDA-event launch time: HBM for the
    bias workload (algorithmic bytes), the bf16 tensor peak otherwise (unmasked
    FLOPs)."""
    fwd_tflops = r["eff_flops"] / (r["ms_fwd"] * 1e-3) / 1e12
    traffic = recorded_traffic(w.name)
    if w.score == "bias":
        achieved = r["alg_bytes"] / (r["ms_fwd"] * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                "peak_source": f"{peak_src} copy bandwidth", "kernel": "flex_fwd_kernel",
                "algorithmic_bytes_per_launch": r["alg_bytes"], "tensor_tflops": round(fwd_tflops, 2)}
    return {"bound": "tensor", "achieved": round(fwd_tflops, 2), "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": round(fwd_tflops / peaks["bf16_tflops"], 4), "traffic": traffic,
            "peak_source": f"{peak_src} bf16 dense burst", "kernel": "flex_fwd_kernel",
            "frac_of_sustained": round(fwd_tflops / peaks["bf16_tflops_sustained"], 4),
            "algorithmic_flops_per_launch": r["eff_flops"]}


def run_ours(args, w, rank, world, dev):
    import block_sparse_attention_48_b200 as fa

    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    r = measure(fa, w, dev, stream, args.steps, args.warmup, world, split_full=not args.no_full, clocks=sampler)
    q_h, k_h, v_h, doc, score_h = r.pop("inputs")
    # end to end through the public API from pinned host buffers
    r["e2e"] = run_e2e(fa, args, w, dev, stream, q_h, k_h, v_h, doc, score_h, r["eff_flops"], world)
    return r


def measure_paged(fa, w, dev, stream, steps, warmup):
    """The forward pass of workload w over a paged KV cache: K and V scattered into
    page pools [B * nkv, Hkv, 128, D] by a seeded permutation, a page table
    [B, nkv]; the forward kernel timed alone (L2 flushed before each launch)."""
    q_h, k_h, v_h = W.qkv(w)
    nkv = (w.kv_len + 127) // 128
    g = torch.Generator().manual_seed(4242)
    perm = torch.randperm(w.B * nkv, generator=g)
    with torch.cuda.stream(stream):
        q = q_h.to(dev)

        def pool(t):
            t = t.to(dev)
            pad = torch.zeros((w.B, w.Hkv, nkv * 128, w.D), dtype=t.dtype, device=dev)
            pad[:, :, : w.kv_len] = t
            blocks = pad.view(w.B, w.Hkv, nkv, 128, w.D).permute(0, 2, 1, 3, 4).reshape(w.B * nkv, w.Hkv, 128, w.D)
            out = torch.empty_like(blocks)
            out[perm.to(dev)] = blocks
            return out

        kp, vp = pool(k_h), pool(v_h)
        pt = perm.view(w.B, nkv).to(torch.int32).to(dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device=dev)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        score = device_score(w, host_score(w), dev)
    stream.synchronize()
    bm = fa.create_block_mask(w.mask_op, list(w.mask_leaves), 1, 1, w.q_len, w.kv_len, stream=stream)
    lib = fa.library()
    qd, kd, vd, od = (fa.tensor_desc(t) for t in (q, kp, vp, o))
    sm, keep = fa.score_mod_desc(score)
    ws = fa.workspace(dev)
    st = ctypes.c_void_p(stream.cuda_stream)

    def fwd():
        rc = lib.fa_forward_paged(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.c_void_p(pt.data_ptr()),
                                  pt.stride(0), ctypes.byref(bm.desc), ctypes.byref(sm), ctypes.c_float(0.0),
                                  ctypes.byref(od), ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                  ctypes.c_size_t(ws.numel()), st)
        if rc:
            raise RuntimeError(fa.status_string(rc))

    for _ in range(warmup):
        with torch.cuda.stream(stream):
            flush.zero_()
        fwd()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        with torch.cuda.stream(stream):
            flush.zero_()
        ev[i][0].record(stream)
        fwd()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    status = fa.device_status(stream=stream)
    if status != 0:
        raise RuntimeError(f"device status {fa.status_string(status)} after the paged forward")
    pairs = admitted_pairs(w, None)
    return dict(ms_fwd=sum(a.elapsed_time(b) for a, b in ev) / steps, eff_flops=4.0 * w.D * pairs,
                alg_bytes=algorithmic_bytes(w, pairs), pairs=pairs)


# Decoding workload: one new token per sequence against a 32k cache, LLaMA-3-8B
# head layout (32 query heads on 8 kv heads, D = 128), causal at the token's
# position.  HBM-bound: K and V of every cached token are read once.
DECODE = dict(name="decode_b8_hq32_hkv8_q1_kv32768_d128", B=8, Hq=32, Hkv=8, q_len=1, kv_len=32768, D=128)


def measure_decode(fa, dev, stream, steps, warmup, peaks, peak_src):
    d = DECODE
    g = torch.Generator().manual_seed(7)
    q = torch.randn((d["B"], d["Hq"], d["q_len"], d["D"]), generator=g).to(torch.bfloat16)
    with torch.cuda.stream(stream):
        q = q.to(dev)
        k = torch.randn((d["B"], d["Hkv"], d["kv_len"], d["D"]), device=dev, dtype=torch.float32).to(torch.bfloat16)
        v = torch.randn_like(k)
        o = torch.empty_like(q)
        lse = torch.empty((d["B"], d["Hq"], d["q_len"]), dtype=torch.float32, device=dev)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream.synchronize()
    off = d["kv_len"] - d["q_len"]
    bm = fa.create_block_mask("and", [("causal",)], 1, 1, d["q_len"], d["kv_len"], q_offset=off, stream=stream)
    lib = fa.library()
    need = int(lib.fa_decode_workspace_size(d["B"], d["Hq"], d["Hkv"], d["q_len"], d["kv_len"], d["D"]))
    ws = torch.zeros((need,), dtype=torch.uint8, device=dev)
    qd, kd, vd, od = (fa.tensor_desc(t) for t in (q, k, v, o))
    sm, keep = fa.score_mod_desc(None)
    st = ctypes.c_void_p(stream.cuda_stream)

    def dec():
        rc = lib.fa_decode(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(bm.desc),
                           ctypes.byref(sm), ctypes.c_float(0.0), ctypes.byref(od), ctypes.c_void_p(lse.data_ptr()),
                           ctypes.c_void_p(ws.data_ptr()), ctypes.c_size_t(ws.numel()), st)
        if rc:
            raise RuntimeError(fa.status_string(rc))

    for _ in range(warmup):
        with torch.cuda.stream(stream):
            flush.zero_()
        dec()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        with torch.cuda.stream(stream):
            flush.zero_()
        ev[i][0].record(stream)
        dec()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    status = fa.device_status(ws=ws, stream=stream)
    if status != 0:
        raise RuntimeError(f"device status {fa.status_string(status)} after decoding")
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    kv_bytes = 2 * d["B"] * d["Hkv"] * d["kv_len"] * d["D"] * 2
    qo_bytes = 2 * d["B"] * d["Hq"] * d["q_len"] * d["D"] * 2 + d["B"] * d["Hq"] * d["q_len"] * 4
    alg = kv_bytes + qo_bytes
    achieved = alg / (ms * 1e-3) / 1e9
    flops = 4.0 * d["D"] * d["B"] * d["Hq"] * d["q_len"] * d["kv_len"]
    return {"decode_ms": round(ms, 5), "steps": steps, "device_status": "FA_OK",
            "workload": dict(d, mask="causal at q_offset = kv_len - 1"),
            "effective_tflops": round(flops / (ms * 1e-3) / 1e12, 3),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": recorded_traffic(d["name"], "flex_decode"),
                         "peak_source": f"{peak_src} copy bandwidth", "kernel": "flex_decode_kernel",
                         "algorithmic_bytes_per_launch": alg}}


def measure_backward(fa, w, dev, stream, steps, warmup, peaks, peak_src):
    """fa_backward of workload w (transposed BlockMask built once): dQ, dK, dV from
    the forward's O and LSE and a seeded dO; timed alone, L2 flushed before each.
    Effective FLOPs: 5 products of 2 * D per admitted pair (S recomputed, dP, dV,
    dK, dQ), i.e. 2.5 times the forward pass."""
    q_h, k_h, v_h = W.qkv(w)
    doc = W.document_ids(w)
    with torch.cuda.stream(stream):
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
        score = device_score(w, host_score(w), dev)
        do = torch.randn(q.shape, device=dev, dtype=torch.float32).to(torch.bfloat16)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        Bm = w.B if w.has_document else 1
    bm = fa.create_block_mask(w.mask_op, list(w.mask_leaves), Bm, 1, w.q_len, w.kv_len, doc_ids=doc, stream=stream,
                              transposed=True)
    with torch.cuda.stream(stream):
        o, lse = fa.flex_attention(q, k, v, bm, score_mod=score, stream=stream)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.zeros((int(fa.library().fa_backward_workspace_size(w.B, w.Hq, w.q_len, w.D)),),
                         dtype=torch.uint8, device=dev)

    def bwd():
        fa.flex_attention_backward(q, k, v, o, lse, do, bm, score_mod=score, dq=dq, dk=dk, dv=dv, ws=ws, stream=stream)

    for _ in range(warmup):
        with torch.cuda.stream(stream):
            flush.zero_()
        bwd()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        with torch.cuda.stream(stream):
            flush.zero_()
        ev[i][0].record(stream)
        bwd()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    status = fa.device_status(ws=ws, stream=stream)
    if status != 0:
        raise RuntimeError(f"device status {fa.status_string(status)} after the backward pass ({w.name})")
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    pairs = admitted_pairs(w, doc)
    flops = 10.0 * w.D * pairs
    tf = flops / (ms * 1e-3) / 1e12
    return {"backward_ms": round(ms, 5), "steps": steps, "device_status": "FA_OK",
            "step": "fa_backward (Delta prologue, tcgen05 kernel, dQ epilogue)",
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(tf / peaks["bf16_tflops"], 4), "traffic": recorded_traffic(w.name, "flex_bwd"),
                         "peak_source": f"{peak_src} bf16 dense burst", "kernel": "flex_bwd_kernel",
                         "algorithmic_flops_per_launch": flops}}


def run_per_config(args, headline, dev, peaks, peak_src):
    """The other workloads (and the headline without the full / partial split),
    measured in the same process: forward-kernel and step time, roofline, device
    status.  One GPU only."""
    import block_sparse_attention_48_b200 as fa

    stream = torch.cuda.Stream(device=dev)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    steps = max(3, min(args.steps, 10))
    jobs = [(i, True) for i in range(len(W.CONFIGS)) if i != headline] + [(headline, False)]
    out = {}
    sampler.start()
    time.sleep(0.3)
    for i, split in jobs:
        w = W.config(i)
        r = measure(fa, w, dev, stream, steps, 3, split_full=split)
        r.pop("inputs")
        key = w.name if split else f"{w.name}__no_full_split"
        out[key] = {"forward_kernel_ms": round(r["ms_fwd"], 5), "step_ms": round(r["ms_step"], 5),
                    "effective_tflops_step": round(r["eff_flops"] / (r["ms_step"] * 1e-3) / 1e12, 3),
                    "unmasked_pairs": r["pairs"], "steps": steps, "device_status": r["status"],
                    "blockmask": "full/partial split" if split else "no split (every tile masked per element)",
                    "roofline": roofline(w, r, peaks, peak_src)}
        torch.cuda.empty_cache()
    # the headline workload over a paged KV cache (kv indices as a page table)
    w = W.config(headline)
    r = measure_paged(fa, w, dev, stream, steps, 3)
    out[f"{w.name}__paged"] = {
        "forward_kernel_ms": round(r["ms_fwd"], 5), "steps": steps, "device_status": "FA_OK",
        "kv_cache": "pages [B*nkv, Hkv, 128, D] in seeded random order, page table [B, nkv]",
        "roofline": roofline(w, r, peaks, peak_src)}
    torch.cuda.empty_cache()
    out[DECODE["name"]] = measure_decode(fa, dev, stream, steps, 3, peaks, peak_src)
    torch.cuda.empty_cache()
    for i in (headline, 2):
        out[f"{W.config(i).name}__backward"] = measure_backward(fa, W.config(i), dev, stream, steps, 3, peaks,
                                                                 peak_src)
        torch.cuda.empty_cache()
    torch.cuda.empty_cache()
    out["clocks"] = sampler.stop()
    return out


def run_e2e(fa, args, w, dev, stream, q_h, k_h, v_h, doc, score_h, eff_flops, world):
    """The headline step through the public Python API with host buffers: every
    step copies its Q, K, V (and bias / slopes) in from pinned host memory, builds
    the BlockMask, runs flex_attention and copies O and LSE back to pinned host
    memory.  Copies in, compute and copies out run on three streams over two
    buffer sets, so that step i + 1's inputs cross the link while step i computes
    and its results cross the other way (the link is full duplex); events order
    every buffer's reuse."""
    pin = lambda t: t.contiguous().pin_memory()
    qp, kp, vp = pin(q_h), pin(k_h), pin(v_h)
    bias_p = pin(score_h[1]) if score_h[0] == "bias" else None
    slopes_p = pin(score_h[1]) if score_h[0] == "alibi" else None
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    sets = []
    for _ in range(2):
        with torch.cuda.stream(stream):
            d = {"q": torch.empty_like(qp, device=dev), "k": torch.empty_like(kp, device=dev),
                 "v": torch.empty_like(vp, device=dev),
                 "bias": torch.empty_like(bias_p, device=dev) if bias_p is not None else None,
                 "slopes": torch.empty_like(slopes_p, device=dev) if slopes_p is not None else None,
                 "o": torch.empty(q_h.shape, dtype=torch.bfloat16, device=dev),
                 "lse": torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device=dev)}
        d["o_host"] = torch.empty(q_h.shape, dtype=torch.bfloat16).pin_memory()
        d["lse_host"] = torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32).pin_memory()
        d["ev_in"], d["ev_comp"], d["ev_out"] = (torch.cuda.Event() for _ in range(3))
        sets.append(d)
    doc_d = doc.to(dev) if doc is not None else None
    h2d = qp.numel() * 2 + kp.numel() * 2 + vp.numel() * 2 + (bias_p.numel() * 2 if bias_p is not None else 0) + \
        (slopes_p.numel() * 4 if slopes_p is not None else 0)
    d2h = sets[0]["o_host"].numel() * 2 + sets[0]["lse_host"].numel() * 4
    Bm = w.B if w.has_document else 1

    def one(i):
        d = sets[i % 2]
        with torch.cuda.stream(s_in):
            s_in.wait_event(d["ev_comp"])  # the set's previous step has read its inputs
            d["q"].copy_(qp, non_blocking=True)
            d["k"].copy_(kp, non_blocking=True)
            d["v"].copy_(vp, non_blocking=True)
            if d["bias"] is not None:
                d["bias"].copy_(bias_p, non_blocking=True)
            if d["slopes"] is not None:
                d["slopes"].copy_(slopes_p, non_blocking=True)
            d["ev_in"].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(d["ev_in"])
            stream.wait_event(d["ev_out"])  # the set's previous results have been copied out
            sm = (("bias", d["bias"]) if d["bias"] is not None else (("alibi", d["slopes"]) if d["slopes"] is not None
                                                                      else (score_h if score_h[0] == "softcap" else None)))
            bm = fa.create_block_mask(w.mask_op, list(w.mask_leaves), Bm, 1, w.q_len, w.kv_len, doc_ids=doc_d,
                                      stream=stream)
            fa.flex_attention(d["q"], d["k"], d["v"], bm, score_mod=sm, out=d["o"], lse=d["lse"], stream=stream)
            d["ev_comp"].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(d["ev_comp"])
            d["o_host"].copy_(d["o"], non_blocking=True)
            d["lse_host"].copy_(d["lse"], non_blocking=True)
            d["ev_out"].record(s_out)

    steps = max(3, min(args.steps, 10))
    for i in range(2):
        one(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        one(i)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks([e0.elapsed_time(e1) / steps], world, dev)[0]
    return {"value": round(aggregate_tflops(eff_flops, world, ms), 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 4),
            "schedule": "copies in, compute and copies out on three streams over two buffer sets"}


# ---------------------------------------------------------------- oracle (CPU baseline / reference arm)

def oracle_sample(w, rows_per_step, seed):
    import oracle
    q, k, v = W.qkv(w)
    doc = W.document_ids(w)
    score = ("alibi", W.alibi_slopes(w.Hq)) if w.score == "alibi" else (
        ("softcap", w.softcap) if w.score == "softcap" else (("bias", W.bias(w, 0)) if w.score == "bias" else ("none",)))
    rows = W.random_rows(w, rows_per_step, seed=seed)
    # effective FLOPs of the sampled rows: admitted keys per row from the mask's closed form
    pairs = 0
    leaves = [l[0] for l in w.mask_leaves]
    ids = doc.tolist() if doc is not None else None
    for b, h, qi in rows.tolist():
        if leaves == ["causal"]:
            pairs += qi + 1
        elif leaves == ["causal", "sliding"]:
            pairs += min(qi, w.mask_leaves[1][1]) + 1
        else:
            j = qi
            while j > 0 and ids[b][j - 1] == ids[b][qi]:
                j -= 1
            pairs += qi - j + 1
    flops = 4.0 * w.D * pairs
    threads = oracle.default_threads()

    def run():
        oracle.forward(q, k, v, w.mask_op, list(w.mask_leaves), doc, score=score, rows=rows, n_threads=threads)

    return run, flops, threads, rows.shape[0]


def rows_for_seconds(w, seconds):
    """Rows of the workload the oracle covers in about `seconds` (a short probe)."""
    import oracle
    run, flops, threads, n = oracle_sample(w, 64, seed=123)
    t0 = time.time()
    run()
    dt = max(time.time() - t0, 1e-3)
    return max(64, int(64 * seconds / dt))


def cpu_baseline(w):
    n = rows_for_seconds(w, 12.0)
    run, flops, threads, n = oracle_sample(w, n, seed=321)
    t0 = time.time()
    run()
    dt = time.time() - t0
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} seeded random query rows of {w.name} (of {w.B * w.Hq * w.q_len}); "
                      f"fp64 dense oracle, {dt:.1f} s"}


def run_reference(args, w, rank, world):
    if rank != 0:
        return None
    n = rows_for_seconds(w, 3.0)
    run, flops, threads, n = oracle_sample(w, n, seed=555)
    for _ in range(args.warmup):
        run()
    times = []
    for _ in range(args.steps):
        t0 = time.time()
        run()
        times.append(time.time() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms * 1e-3) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.q_len, "D": w.D,
                       "mask": "+".join(l[0] for l in w.mask_leaves), "score_mod": w.score,
                       "sample_rows_per_step": n},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n} seeded random query rows per step of {w.name}"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


# ---------------------------------------------------------------- main

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=1, help="index into workloads.CONFIGS (1 = headline)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="skip the other workloads (per_config key)")
    ap.add_argument("--no-full", action="store_true",
                    help="headline without the full / partial split (every listed tile masked per element)")
    ap.add_argument("--kernel", choices=["forward", "backward", "decode", "paged"], default="forward",
                    help="backward / decode / paged: time only that path on the --config workload (decode: its own "
                         "workload) and print its per_config entry; for profiling single kernels")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = W.config(args.config)

    if args.impl == "reference":
        line = run_reference(args, w, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    dev = torch.device("cuda", local)
    if args.kernel != "forward":
        import block_sparse_attention_48_b200 as fa
        torch.cuda.set_device(dev)
        stream = torch.cuda.Stream(device=dev)
        peaks, peak_src = load_peaks()
        if args.kernel == "backward":
            entry = measure_backward(fa, w, dev, stream, args.steps, args.warmup, peaks, peak_src)
        elif args.kernel == "decode":
            entry = measure_decode(fa, dev, stream, args.steps, args.warmup, peaks, peak_src)
        else:
            r = measure_paged(fa, w, dev, stream, args.steps, args.warmup)
            entry = {"forward_kernel_ms": round(r["ms_fwd"], 5), "roofline": roofline(w, r, peaks, peak_src)}
        print(json.dumps({"kernel": args.kernel, "workload": DECODE["name"] if args.kernel == "decode" else w.name,
                          **entry}), flush=True)
        return 0
    if world > 1:
        import datetime
        torch.cuda.set_device(dev)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    r = run_ours(args, w, rank, world, dev)
    peaks, peak_src = load_peaks()
    if rank == 0:
        value = aggregate_tflops(r["eff_flops"], world, r["ms_step"])
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(r["ms_step"], 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.q_len, "D": w.D,
                       "mask": "+".join(l[0] for l in w.mask_leaves), "score_mod": w.score,
                       "unmasked_pairs": r["pairs"], "parallelism": f"replicas{world}",
                       "l2": "flushed between timed steps (256 MiB write, outside the events)",
                       "step": "fa_create_block_mask + fa_forward" if not args.no_full
                       else "fa_create_block_mask_unsplit + fa_forward"},
            "pct_of_bf16_peak": round(100 * value / world / peaks["bf16_tflops"], 2),
            "forward_kernel_ms": round(r["ms_fwd"], 5),
            "roofline": roofline(w, r, peaks, peak_src),
            "e2e": r["e2e"],
            "gpu_launches": 2 * args.steps,
            "clocks": r["clocks"],
        }
        if world == 1 and not args.no_per_config:
            pc = run_per_config(args, args.config, dev, peaks, peak_src)
            paged = pc.get(f"{w.name}__paged")
            if paged:
                paged["vs_contiguous_forward"] = round(paged["forward_kernel_ms"] / r["ms_fwd"], 4)
            line["per_config"] = pc
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

"""The decode kernel's walk over the list of kv blocks (csrc/decode_walk.cuh),
built for the host ("Flex Attention" paper review sec. 3.1, the decoding
template: the work split along the KV dimension).  The list holds every
(batch, kv head) segment's BlockMask row, partial blocks first; CTA c of G takes
entries [floor(c T / G), floor((c + 1) T / G)).  With the kernel's start-up step
reproduced here (a scan of the rows' block counts over the CTA's threads, then
the thread whose rows hold the share's first entry finds its position), every
entry must go to exactly one CTA, in list order and with its BlockMask index;
the partial results numbered (segment + CTA) must be distinct and inside the
workspace; and the merge's view of a segment (the CTAs from the holder of its
first block to the holder of its last, less those with an empty share) must be
exactly the CTAs that hold its blocks."""

import ctypes
import os
import random
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "host", "decode_walk.cpp")
BUILD = os.path.join(ROOT, "tests", "host", "_build")
LIB = os.path.join(BUILD, "libdecodewalk.so")
THREADS = 288  # a decode CTA: eight compute warps and the TMA producer warp

I32P = ctypes.POINTER(ctypes.c_int32)


@pytest.fixture(scope="module")
def lib():
    os.makedirs(BUILD, exist_ok=True)
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(ROOT, "block_sparse_attention_48_b200", "csrc"), SRC, "-o", LIB])
    L = ctypes.CDLL(LIB)
    L.fa_host_share_start.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_int]
    L.fa_host_share_start.restype = ctypes.c_longlong
    L.fa_host_dec_find.argtypes = [ctypes.c_int32] * 5 + [I32P, I32P, ctypes.c_longlong, ctypes.c_int, ctypes.c_int,
                                                          ctypes.c_longlong, I32P]
    L.fa_host_dec_find_shared.argtypes = [ctypes.c_int32] * 4 + [I32P, I32P, ctypes.c_longlong, ctypes.c_longlong,
                                                                 I32P]
    L.fa_host_dec_walk.argtypes = [ctypes.c_int32] * 5 + [I32P] * 4 + [ctypes.c_int] * 3 + [ctypes.c_longlong, I32P]
    return L


def ptr(a):
    return a.ctypes.data_as(I32P)


def make_mask(rng, nrow, nkv, has_full):
    """Random BlockMask rows: disjoint partial and full lists of distinct blocks,
    some rows empty."""
    kv_num = np.zeros(nrow, np.int32)
    full_num = np.zeros(nrow, np.int32)
    kv_idx = np.zeros((nrow, max(nkv, 1)), np.int32)
    full_idx = np.zeros((nrow, max(nkv, 1)), np.int32)
    for r in range(nrow):
        mode = rng.random()
        n = 0 if mode < 0.2 else (nkv if mode < 0.5 else rng.randint(0, nkv))
        blocks = rng.sample(range(nkv), n)
        nf = rng.randint(0, n) if has_full else 0
        kv_num[r], full_num[r] = n - nf, nf
        kv_idx[r, : n - nf] = blocks[: n - nf]
        full_idx[r, :nf] = blocks[n - nf:]
    return kv_num, full_num, kv_idx, full_idx


def run_case(lib, rng, B, Hkv, nkv, bm_b1, has_full, G):
    nrow = 1 if bm_b1 else B
    kv_num, full_num, kv_idx, full_idx = make_mask(rng, nrow, nkv, has_full)
    cnt = (kv_num + full_num).astype(np.int64)
    # the list, entry by entry: (b, hk, t, kv block)
    entries = []
    for b in range(B):
        r = 0 if bm_b1 else b
        for hk in range(Hkv):
            for t in range(int(cnt[r])):
                kb = kv_idx[r, t] if t < kv_num[r] else full_idx[r, t - kv_num[r]]
                entries.append((b, hk, t, int(kb)))
    # the start-up scan: thread i sums rows [i per, (i + 1) per)
    per = (nrow + THREADS - 1) // THREADS
    ranges = [(min(nrow, i * per), min(nrow, min(nrow, i * per) + per)) for i in range(THREADS)]
    mine = [int(cnt[lo:hi].sum()) for lo, hi in ranges]
    excl = np.concatenate([[0], np.cumsum(mine)[:-1]]).astype(np.int64)
    total = int(sum(mine))
    T = Hkv * (total * B if bm_b1 else total)
    assert T == len(entries)
    out = np.zeros(5, np.int32)
    owner = {}
    holders = {}
    pieces = set()
    first_holder, last_holder = {}, {}
    for c in range(G):
        x0, x1 = lib.fa_host_share_start(T, c, G), lib.fa_host_share_start(T, c + 1, G)
        assert 0 <= x0 <= x1 <= T
        if x0 == x1:
            continue
        if bm_b1:
            lib.fa_host_dec_find_shared(B, Hkv, nkv, int(has_full), ptr(kv_num), ptr(full_num), x0, total, ptr(out))
        else:
            finders = [i for i in range(THREADS) if Hkv * excl[i] <= x0 < Hkv * (excl[i] + mine[i])]
            assert len(finders) == 1
            i = finders[0]
            rc = lib.fa_host_dec_find(B, Hkv, nkv, 0, int(has_full), ptr(kv_num), ptr(full_num), x0, ranges[i][0],
                                      ranges[i][1], int(excl[i]), ptr(out))
            assert rc == 1
        b, hk, t = int(out[0]), int(out[1]), int(out[2])
        count = x1 - x0
        walk = np.zeros(5 * count, np.int32)
        rc = lib.fa_host_dec_walk(B, Hkv, nkv, int(bm_b1), int(has_full), ptr(kv_num), ptr(full_num), ptr(kv_idx),
                                  ptr(full_idx), b, hk, t, count, ptr(walk))
        assert rc == 0
        w = walk.reshape(count, 5)
        for j in range(count):
            got = (int(w[j, 0]), int(w[j, 1]), int(w[j, 2]), int(w[j, 4]))
            assert got == entries[x0 + j], (c, j, got, entries[x0 + j])
            assert (x0 + j) not in owner
            owner[x0 + j] = c
            seg = got[0] * Hkv + got[1]
            holders.setdefault(seg, set()).add(c)
            if got[2] == 0:
                first_holder[seg] = c
            r = 0 if bm_b1 else got[0]
            if got[2] + 1 == cnt[r]:
                last_holder[seg] = c
            pieces.add((seg, c))
    assert len(owner) == T
    # partial results: number segment + CTA, distinct, inside [0, B Hkv + G)
    numbers = [seg + c for seg, c in pieces]
    assert len(set(numbers)) == len(numbers) and all(0 <= n < B * Hkv + G for n in numbers)
    # the merge's view of each non-empty segment
    for seg, hs in holders.items():
        view = {c for c in range(first_holder[seg], last_holder[seg] + 1)
                if lib.fa_host_share_start(T, c, G) < lib.fa_host_share_start(T, c + 1, G)}
        assert view == hs, (seg, sorted(view), sorted(hs))


def test_share_start_is_exact_floor_division(lib):
    rng = random.Random(5)
    for _ in range(2000):
        T = rng.choice([0, 1, 7, 147, 148, 149, rng.randint(0, 10**6), rng.randint(0, 2**60)])
        G = rng.choice([1, 2, 148, 300])
        c = rng.randint(0, G)
        assert lib.fa_host_share_start(T, c, G) == c * T // G


@pytest.mark.parametrize("seed", range(6))
def test_walk_gives_every_entry_to_one_cta(lib, seed):
    rng = random.Random(100 + seed)
    for _ in range(40):
        B = rng.choice([1, 2, 3, 8, 17, 300, 700])
        Hkv = rng.choice([1, 2, 8])
        nkv = rng.choice([1, 2, 5, 40])
        run_case(lib, rng, B, Hkv, nkv, rng.random() < 0.3, rng.random() < 0.7, rng.choice([1, 2, 7, 148, 300]))


def test_corrupt_counts_are_clamped_and_reported(lib):
    """A count outside [0, nkv] is clamped (the kernel reports FA_ERR_BAD_BLOCKMASK)."""
    kv_num = np.array([5, -3], np.int32)
    full_num = np.array([9, 0], np.int32)
    out = np.zeros(5, np.int32)
    rc = lib.fa_host_dec_find(2, 1, 4, 0, 1, ptr(kv_num), ptr(full_num), 0, 0, 2, 0, ptr(out))
    assert rc == 3 and out[3] == 4 and out[4] == 8  # found, with the counts clamped to nkv

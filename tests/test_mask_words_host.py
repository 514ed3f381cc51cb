"""The device mask logic of csrc/mask_eval.cuh, built for the host: the forward
kernel's per-row mask words and the BlockMask build's tile summaries, checked
against the leaf definitions evaluated position by position ("Concepts",
mask_mod and Composing masks): causal q >= kv, sliding q - kv <= W, prefix
kv < P, document doc[q] == doc[kv], kv < kv_len, combined by one AND or OR."""

import ctypes
import os
import random
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "host", "mask_words.cpp")
BUILD = os.path.join(ROOT, "tests", "host", "_build")
LIB = os.path.join(BUILD, "libmaskwords.so")

CAUSAL, SLIDING, DOCUMENT, PREFIX = 0, 1, 2, 3
AND, OR = 0, 1


@pytest.fixture(scope="module")
def lib():
    os.makedirs(BUILD, exist_ok=True)
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(ROOT, "block_sparse_attention_48_b200", "csrc"), SRC, "-o", LIB])
    L = ctypes.CDLL(LIB)
    L.fa_host_row_mask.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int32),
                                   ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint32)]
    return L


def words(lib, leaves, op, q, k0, kv_len, dbits):
    kind = (ctypes.c_int32 * 4)(*([k for k, _ in leaves] + [0] * (4 - len(leaves))))
    param = (ctypes.c_int64 * 4)(*([p for _, p in leaves] + [0] * (4 - len(leaves))))
    d = (ctypes.c_uint32 * 4)(*dbits)
    out = (ctypes.c_uint32 * 4)()
    lib.fa_host_row_mask(len(leaves), op, kind, param, q, k0, kv_len, d, out)
    return list(out)


def expected(leaves, op, q, k0, kv_len, dbits):
    w = [0, 0, 0, 0]
    for c in range(128):
        kv = k0 + c
        vals = []
        for kind, prm in leaves:
            if kind == CAUSAL:
                vals.append(q >= kv)
            elif kind == SLIDING:
                vals.append(q - kv <= prm)
            elif kind == PREFIX:
                vals.append(kv < prm)
            else:
                vals.append(bool((dbits[c >> 5] >> (c & 31)) & 1))
        ok = (any(vals) if op == OR else all(vals)) if leaves else True
        if ok and kv < kv_len:
            w[c >> 5] |= 1 << (c & 31)
    return w


def random_case(rng):
    n = rng.randint(0, 4)
    leaves = []
    for _ in range(n):
        kind = rng.choice([CAUSAL, SLIDING, DOCUMENT, PREFIX])
        if kind == SLIDING:
            prm = rng.choice([0, 1, 5, 100, 127, 128, 1024, 2 ** 31, 2 ** 40, -3])
        elif kind == PREFIX:
            prm = rng.choice([-5, 0, 1, 64, 200, 5000, 2 ** 31 - 1, 2 ** 62])
        else:
            prm = 0
        leaves.append((kind, prm))
    op = rng.choice([AND, OR])
    k0 = 128 * rng.randint(0, 40)
    q = k0 + rng.randint(-300, 300)
    q = max(q, 0)
    kv_len = k0 + rng.choice([1, 7, 64, 127, 128, 129, 4000])
    dbits = [rng.getrandbits(32) for _ in range(4)]
    return leaves, op, q, k0, kv_len, dbits


def test_row_mask_words_match_the_leaf_definitions(lib):
    rng = random.Random(20261202)
    for _ in range(3000):
        leaves, op, q, k0, kv_len, dbits = random_case(rng)
        want = expected(leaves, op, q, k0, kv_len, dbits)
        got = words(lib, leaves, op, q, k0, kv_len, dbits)
        assert got == want, (leaves, op, q, k0, kv_len)


def test_large_positions_and_parameters(lib):
    """Positions near the 2^31 length bound and window / prefix parameters far
    outside int32: the 32-bit tile-local arithmetic must clamp, not wrap."""
    big = 2 ** 31 - 512
    cases = [
        ([(SLIDING, 2 ** 40)], AND, big, big - 128, big + 100),
        ([(SLIDING, 2 ** 40), (CAUSAL, 0)], AND, big, big, big + 128),
        ([(PREFIX, 2 ** 62)], OR, 5, big - 128, big),
        ([(PREFIX, -(2 ** 40))], OR, 5, 0, 128),
        ([(CAUSAL, 0)], AND, 0, big - 128, big),
        ([(SLIDING, -(2 ** 40))], AND, big, 0, 128),
    ]
    for leaves, op, q, k0, kv_len in cases:
        d = [0xFFFFFFFF] * 4
        want = expected(leaves, op, q, k0, kv_len, d)
        assert words(lib, leaves, op, q, k0, kv_len, d) == want, (leaves, q, k0)


def test_tile_summaries_are_sound(lib):
    """The BlockMask build's per-tile summary (all masked / all admitted /
    undecided, from interval bounds and document-id ranges) never claims a
    decision that the element-wise mask contradicts, and decides a single
    interval leaf exactly."""
    f = lib.fa_host_mask_summary
    f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)] + \
        [ctypes.c_int64] * 4 + [ctypes.c_int32] * 4
    f.restype = ctypes.c_int
    rng = random.Random(7)
    for _ in range(1500):
        L = 64
        # sorted document ids over positions 0..L-1
        doc, d = [], 0
        for _i in range(L):
            if rng.random() < 0.08:
                d += 1
            doc.append(d)
        leaves = []
        for _l in range(rng.randint(1, 3)):
            kind = rng.choice([CAUSAL, SLIDING, DOCUMENT, PREFIX])
            prm = rng.randint(-4, 70) if kind in (SLIDING, PREFIX) else 0
            leaves.append((kind, prm))
        op = rng.choice([AND, OR])
        q0 = rng.randint(0, L - 1); q1 = rng.randint(q0, min(L - 1, q0 + 20))
        k0 = rng.randint(0, L - 1); k1 = rng.randint(k0, min(L - 1, k0 + 20))
        truth = set()
        for q in range(q0, q1 + 1):
            for kv in range(k0, k1 + 1):
                vals = []
                for kind, prm in leaves:
                    vals.append({CAUSAL: q >= kv, SLIDING: q - kv <= prm, PREFIX: kv < prm,
                                 DOCUMENT: doc[q] == doc[kv]}[kind])
                truth.add(any(vals) if op == OR else all(vals))
        kind = (ctypes.c_int32 * 4)(*([k for k, _ in leaves] + [0] * (4 - len(leaves))))
        param = (ctypes.c_int64 * 4)(*([p for _, p in leaves] + [0] * (4 - len(leaves))))
        s = f(len(leaves), op, kind, param, q0, q1, k0, k1, min(doc[q0:q1 + 1]), max(doc[q0:q1 + 1]),
              min(doc[k0:k1 + 1]), max(doc[k0:k1 + 1]))
        if s == 1:
            assert truth == {True}, (leaves, op, q0, q1, k0, k1)
        elif s == 0:
            assert truth == {False}, (leaves, op, q0, q1, k0, k1)
        else:
            assert s == 2
            if len(leaves) == 1 and leaves[0][0] != DOCUMENT:
                assert truth == {True, False}, (leaves, q0, q1, k0, k1)


def test_col_mask_words_match_the_leaf_definitions(lib):
    """The backward pass's transposed words: for key kv, bit c of word j is the
    mask at query q0 + 32 j + c, ANDed with q < q_len."""
    f = lib.fa_host_col_mask
    f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64),
                  ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(ctypes.c_uint32),
                  ctypes.POINTER(ctypes.c_uint32)]
    rng = random.Random(20261203)
    for _ in range(3000):
        leaves, op, q, k0, kv_len, dbits = random_case(rng)
        # reuse the generator: here k0 plays the query block start, q the key
        q0, kv, q_len = k0, q, kv_len
        want = [0, 0, 0, 0]
        for c in range(128):
            qq = q0 + c
            vals = []
            for kind, prm in leaves:
                if kind == CAUSAL:
                    vals.append(qq >= kv)
                elif kind == SLIDING:
                    vals.append(qq - kv <= prm)
                elif kind == PREFIX:
                    vals.append(kv < prm)
                else:
                    vals.append(bool((dbits[c >> 5] >> (c & 31)) & 1))
            ok = (any(vals) if op == OR else all(vals)) if leaves else True
            if ok and qq < q_len:
                want[c >> 5] |= 1 << (c & 31)
        kind = (ctypes.c_int32 * 4)(*([k for k, _ in leaves] + [0] * (4 - len(leaves))))
        param = (ctypes.c_int64 * 4)(*([p for _, p in leaves] + [0] * (4 - len(leaves))))
        d = (ctypes.c_uint32 * 4)(*dbits)
        out = (ctypes.c_uint32 * 4)()
        f(len(leaves), op, kind, param, kv, q0, q_len, d, out)
        assert list(out) == want, (leaves, op, kv, q0, q_len)

"""Prefix-hash block manager (MapFlow section 5.3, "Block Manager"): host-only checks.

The manager indexes whole-block token prefixes and hands back the stored per-layer map
descriptors whose leading query blocks a request can reuse.  It never touches device memory, so
these tests give it descriptors with placeholder pointers.
"""
import ctypes
import threading

import numpy as np
import pytest


@pytest.fixture(scope="module")
def mr():
    from cross_model_attention_mr_b200 import mr as m
    return m


B = 64


def _maps(mr, n_layers, L, tag):
    # descriptors only: the pointers are labels the manager must hand back unchanged
    return (mr.BSR * n_layers)(*[mr.BSR(4, L, B, 0, 10, tag + 16 * l, tag + 16 * l + 1, tag + 16 * l + 2,
                                        tag + 16 * l + 3, tag + 16 * l + 4, None, None, tag + 16 * l + 5)
                                 for l in range(n_layers)])


def _tok(rng, n):
    return np.ascontiguousarray(rng.integers(0, 50000, size=n), dtype=np.int32)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _lookup(mr, bm, tok):
    e = ctypes.c_int64(-7)
    k = mr.LIB.mr_bm_lookup(bm, _p(tok), int(tok.shape[0]), ctypes.byref(e))
    return k, e.value


def test_longest_prefix_in_whole_blocks(mr):
    lib = mr.LIB
    rng = np.random.default_rng(1)
    bm = lib.mr_bm_create(B, 0)
    try:
        a = _tok(rng, 10 * B + 17)                     # 10 whole blocks and a partial one
        ea = lib.mr_bm_insert(bm, _p(a), a.shape[0], _maps(mr, 2, 11 * B, 0x1000), 2, 1000)
        assert ea >= 0
        # same first 5 blocks, then different tokens
        q = np.concatenate([a[: 5 * B], _tok(rng, 3 * B)])
        assert _lookup(mr, bm, q) == (5, ea)
        # a change in the last token of block 3 stops the match after 3 blocks
        q2 = a[: 8 * B].copy()
        q2[4 * B - 1] += 1
        assert _lookup(mr, bm, q2) == (3, ea)
        # a different first block: nothing to reuse
        assert _lookup(mr, bm, _tok(rng, 4 * B)) == (0, -1)
        # the partial last block of the stored sequence is not indexed
        assert _lookup(mr, bm, a) == (10, ea)
        # fewer tokens than a block
        assert _lookup(mr, bm, a[: B - 1]) == (0, -1)
        # the descriptor of layer 1 comes back unchanged
        d = mr.BSR()
        assert lib.mr_bm_map(bm, ea, 1, ctypes.byref(d)) == mr.MR_OK
        assert d.vals == 0x1000 + 16 + 2 and d.L == 11 * B and d.block == B
        assert lib.mr_bm_map(bm, ea, 2, ctypes.byref(d)) == mr.MR_ERR_INVALID_ARG
        st = (ctypes.c_int64 * 5)()
        assert lib.mr_bm_stats(bm, st) == mr.MR_OK
        assert list(st) == [1, 1000, 5, 3, 5 + 3 + 10]
    finally:
        lib.mr_bm_destroy(bm)


def test_longer_and_more_recent_entries_win(mr):
    lib = mr.LIB
    rng = np.random.default_rng(2)
    bm = lib.mr_bm_create(B, 0)
    try:
        base = _tok(rng, 6 * B)
        short = base[: 3 * B]
        long_ = np.concatenate([base, _tok(rng, 2 * B)])
        e1 = lib.mr_bm_insert(bm, _p(short), short.shape[0], _maps(mr, 1, 3 * B, 0x100), 1, 10)
        e2 = lib.mr_bm_insert(bm, _p(long_), long_.shape[0], _maps(mr, 1, 8 * B, 0x200), 1, 10)
        assert _lookup(mr, bm, base[: 2 * B]) == (2, e2)      # both hold it: the most recent one
        assert _lookup(mr, bm, base) == (6, e2)               # only the longer entry holds 6 blocks
        e3 = lib.mr_bm_insert(bm, _p(short), short.shape[0], _maps(mr, 1, 3 * B, 0x300), 1, 10)
        assert _lookup(mr, bm, base[: 3 * B]) == (3, e3)
        assert _lookup(mr, bm, base[: 5 * B]) == (5, e2)
    finally:
        lib.mr_bm_destroy(bm)


def test_budget_evicts_least_recent_unreferenced_entries(mr):
    lib = mr.LIB
    rng = np.random.default_rng(3)
    bm = lib.mr_bm_create(B, 250)
    try:
        toks = [_tok(rng, 2 * B) for _ in range(5)]
        ins = lambda i: lib.mr_bm_insert(bm, _p(toks[i]), toks[i].shape[0], _maps(mr, 1, 2 * B, 0x10 * (i + 1)), 1, 100)
        ids = [ins(i) for i in range(4)]
        # every insert holds a reference: nothing can be evicted yet although 400 > 250 bytes
        out = (ctypes.c_int64 * 8)()
        assert lib.mr_bm_evicted(bm, out, 8) == 0
        # releasing the oldest entries lets the budget take them, oldest first, until it holds
        for e in ids:
            assert lib.mr_bm_release(bm, e) == mr.MR_OK
        n = lib.mr_bm_evicted(bm, out, 8)
        assert list(out[:n]) == [ids[0], ids[1]]
        assert _lookup(mr, bm, toks[1]) == (0, -1)            # gone from the index
        assert lib.mr_bm_release(bm, ids[1]) == mr.MR_ERR_INVALID_ARG   # evicted ids are unknown
        # a lookup makes entry 2 the most recent, so the next insert pushes out entry 3
        assert _lookup(mr, bm, toks[2]) == (2, ids[2])
        assert lib.mr_bm_release(bm, ids[2]) == mr.MR_OK
        e4 = ins(4)
        n = lib.mr_bm_evicted(bm, out, 8)
        assert list(out[:n]) == [ids[3]]
        st = (ctypes.c_int64 * 5)()
        lib.mr_bm_stats(bm, st)
        assert st[0] == 2 and st[1] == 200
        assert _lookup(mr, bm, toks[4]) == (2, e4)
    finally:
        lib.mr_bm_destroy(bm)


def test_rejects_bad_arguments(mr):
    lib = mr.LIB
    assert not lib.mr_bm_create(0, 0)
    assert not lib.mr_bm_create(B, -1)
    bm = lib.mr_bm_create(B, 0)
    try:
        t = np.zeros(B, np.int32)
        assert lib.mr_bm_insert(bm, _p(t), B - 1, _maps(mr, 1, B, 1), 1, 0) == -mr.MR_ERR_INVALID_ARG
        bad = mr.BSR(4, B, 128, 0, 1, 1, 1, 1, 1, 1, None, None, 1)     # another block size
        assert lib.mr_bm_insert(bm, _p(t), B, ctypes.byref(bad), 1, 0) == -mr.MR_ERR_INVALID_ARG
        assert lib.mr_bm_insert(bm, _p(t), B, _maps(mr, 1, B, 1), 0, 0) == -mr.MR_ERR_INVALID_ARG
        e = ctypes.c_int64(0)
        assert lib.mr_bm_lookup(bm, None, -1, ctypes.byref(e)) == -mr.MR_ERR_INVALID_ARG
        assert lib.mr_bm_release(bm, 12345) == mr.MR_ERR_INVALID_ARG
    finally:
        lib.mr_bm_destroy(bm)


def test_concurrent_lookups_and_inserts(mr):
    """ctypes calls release the GIL: threads hit the manager at the same time."""
    lib = mr.LIB
    rng = np.random.default_rng(4)
    bm = lib.mr_bm_create(B, 0)
    seqs = [_tok(rng, 4 * B) for _ in range(8)]
    errors = []

    def worker(w):
        try:
            for it in range(200):
                s = seqs[(w + it) % len(seqs)]
                if it % 10 == 0:
                    e = lib.mr_bm_insert(bm, _p(s), s.shape[0], _maps(mr, 1, 4 * B, 0x40 * (w + 1)), 1, 1)
                    lib.mr_bm_release(bm, e)
                k, e = _lookup(mr, bm, s)
                if e >= 0:
                    assert k == 4
                    lib.mr_bm_release(bm, e)
        except Exception as ex:  # noqa: BLE001
            errors.append(ex)

    th = [threading.Thread(target=worker, args=(w,)) for w in range(8)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    lib.mr_bm_destroy(bm)
    assert not errors

"""Pins for the oracle's copy-on-write block copy: the first page's beam-search
example (§3.5), brute force against numpy fancy indexing, and the rules the
fifth page states for shared blocks (§2.3: copy before writing into a shared
block, refcounts return unreferenced blocks to the free pool)."""

import json
import os

import numpy as np
import pytest


def _example(golden_dir):
    with open(os.path.join(golden_dir, "cow_beam_example.json")) as f:
        return json.load(f)


def _rows(seed, T, Hk, d):
    rng = np.random.default_rng(seed)
    # distinct finite f16 bit patterns (exponent field never all-ones)
    return rng.integers(0, 0x7BFF, size=(T, Hk, d), dtype=np.uint16)


def test_cow_beam_search_example(orc, golden_dir):
    """One sequence of 40 tokens in blocks [0, 1, 2] forks into two beam
    candidates that append different tokens at position 40.  Copy-on-write
    gives the page's tables, one new block, and each candidate sees the
    shared history plus its own token."""
    ex = _example(golden_dir)
    B, Hk, d, nb, L = ex["block_size"], 2, 8, 8, 40
    orig = np.array(ex["original_table"], np.int32)
    kc = orc.empty_pool(nb, Hk, B, d, "f16")
    vc = orc.empty_pool(nb, Hk, B, d, "f16")
    krows, vrows = _rows(1, L, Hk, d), _rows(2, L, Hk, d)
    slots = orc.slot_mapping(orig[None, :], None, np.zeros(L, np.int32),
                             np.arange(L, dtype=np.int32), L, B)
    assert orc.cache_write(krows, vrows, kc, vc, slots, nb, Hk, d, B, "f16", "f16") == 0
    before = kc.copy(), vc.copy()

    # fork: both candidates reference the original blocks
    tables = [orig.copy(), orig.copy()]
    refcount = np.zeros(nb, np.int32)
    for t in tables:
        refcount[t] += 1
    free = [b for b in range(nb) if refcount[b] == 0]
    copies = []
    new_k, new_v = _rows(3, 2, Hk, d), _rows(4, 2, Hk, d)
    # candidate 2 writes first: its target block is shared, so copy it first
    for cand in (1, 0):
        lb = L // B
        phys = int(tables[cand][lb])
        if refcount[phys] > 1:
            fresh = free.pop(0)
            copies.append((phys, fresh))
            assert orc.copy_blocks(kc, vc, np.array([[phys, fresh]], np.int32)) == 0
            refcount[phys] -= 1
            refcount[fresh] += 1
            tables[cand][lb] = fresh
        sl = orc.slot_mapping(tables[cand][None, :], None, np.zeros(1, np.int32),
                              np.array([L], np.int32), 1, B)
        assert orc.cache_write(new_k[cand:cand + 1], new_v[cand:cand + 1], kc, vc, sl, nb, Hk, d,
                               B, "f16", "f16") == 0

    assert [list(t) for t in tables] == ex["candidate_tables"]
    assert [dst for _, dst in copies] == ex["new_blocks"]
    # blocks 0 and 1 stay shared and unchanged
    for b in ex["original_table"][:2]:
        assert refcount[b] == 2
        assert np.array_equal(kc[b], before[0][b]) and np.array_equal(vc[b], before[1][b])
    # memory: 4 distinct blocks instead of 3 x 2; copying: 1 block of 3
    distinct = {int(b) for t in tables for b in t}
    assert len(distinct) == 4 < ex["traditional_blocks"]
    saved = len(ex["original_table"]) - len(copies)
    assert saved * ex["copy_saving"][1] == ex["copy_saving"][0] * len(ex["original_table"])
    # each candidate reads the shared history and then its own token
    for cand in (0, 1):
        for pool, rows, new in ((kc, krows, new_k), (vc, vrows, new_v)):
            for h in range(Hk):
                g = orc.gather(pool, "f16", 1.0, tables[cand], L + 1, Hk, h, d, B)
                want = np.concatenate([rows[:, h, :], new[cand:cand + 1, h, :]])
                assert np.array_equal(g, want.view(np.float16).astype(np.float64))


@pytest.mark.parametrize("kv", ["f16", "e4m3"])
def test_copy_blocks_brute_force(orc, kv):
    """Random disjoint (src, dst) pairs against numpy fancy indexing, over
    pools of distinct bytes; unlisted blocks and both pools checked."""
    rng = np.random.default_rng(7 if kv == "f16" else 8)
    nb, Hk, B, d = 40, 3, 16, 16
    dt = np.uint8 if kv == "e4m3" else np.uint16
    kc = rng.integers(0, np.iinfo(dt).max, size=(nb, Hk, B, d), dtype=dt)
    vc = rng.integers(0, np.iinfo(dt).max, size=(nb, Hk, B, d), dtype=dt)
    ids = rng.permutation(nb)
    src, dst = ids[:12], ids[12:24]
    pairs = np.stack([src, dst], 1).astype(np.int32)
    want_k, want_v = kc.copy(), vc.copy()
    want_k[dst] = kc[src]
    want_v[dst] = vc[src]
    assert orc.copy_blocks(kc, vc, pairs) == 0
    assert np.array_equal(kc, want_k) and np.array_equal(vc, want_v)


def test_copy_blocks_out_of_range_skipped(orc):
    nb, Hk, B, d = 6, 1, 16, 8
    kc = orc.empty_pool(nb, Hk, B, d, "bf16", fill=0x11)
    vc = orc.empty_pool(nb, Hk, B, d, "bf16", fill=0x22)
    kc[2] = 5
    before = kc.copy(), vc.copy()
    pairs = np.array([[2, 6], [-1, 3], [2, -4], [7, 0]], np.int32)
    assert orc.copy_blocks(kc, vc, pairs) == 4
    assert np.array_equal(kc, before[0]) and np.array_equal(vc, before[1])
    assert orc.copy_blocks(kc, vc, np.array([[2, 4], [3, 3]], np.int32)) == 0
    assert np.array_equal(kc[4], before[0][2]) and np.array_equal(kc[3], before[0][3])

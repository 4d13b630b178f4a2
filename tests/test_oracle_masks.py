"""Pins of the oracle's valid-path masks (CPU only).

Definition pinned: xGR page, 2.2 xBeam, "Valid-path constraint" -- the valid
next tokens of a prefix come from a pre-built vocabulary of valid items;
"Hybrid dense/sparse storage" -- a dense mask for the first step, sparse rows
afterwards.
"""
import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_tiny_vocabulary(orc):
    fx = json.load(open(os.path.join(GOLDEN, "mask_tiny.json")))
    items = np.array(fx["items"], np.int32)
    V = fx["V"]
    assert orc.mask_dense(items, V).tolist() == fx["dense_words"]
    si = orc.SortedItems(items, V)
    for case in fx["next"]:
        assert orc.next_tokens_scan(items, case["prefix"], V).tolist() == case["tokens"]
        assert si.next_tokens(case["prefix"]).tolist() == case["tokens"]


def _random_items(seed, n, L, V):
    rng = np.random.default_rng(seed)
    codes = rng.choice(V ** L, size=n, replace=False)
    out = np.zeros((n, L), np.int32)
    for j in range(L - 1, -1, -1):
        out[:, j] = codes % V
        codes //= V
    return out


def test_sorted_lookup_equals_brute_force_scan(orc):
    for seed, (n, L, V) in enumerate([(60, 3, 5), (500, 3, 16), (300, 4, 6)]):
        items = _random_items(seed, n, L, V)
        si = orc.SortedItems(items, V)
        rng = np.random.default_rng(100 + seed)
        prefixes = [items[i, :s] for i in range(0, n, 7) for s in range(L)]
        prefixes += [rng.integers(0, V, size=s) for s in range(L) for _ in range(20)]
        for p in prefixes:
            a = orc.next_tokens_scan(items, p, V)
            b = si.next_tokens(p)
            assert a.tolist() == b.tolist()


def test_every_listed_token_extends_to_an_item_and_none_is_missed(orc):
    items = _random_items(7, 400, 3, 12)
    V = 12
    pre = {tuple(it[:s]) for it in items.tolist() for s in range(4)}
    si = orc.SortedItems(items, V)
    for p in [(), (3,), (5, 1), (11,), (0, 0)]:
        got = set(si.next_tokens(list(p)).tolist())
        want = {t for t in range(V) if tuple(p) + (t,) in pre}
        assert got == want


def test_dense_bits_are_first_tokens(orc):
    items = _random_items(9, 200, 3, 70)
    bits = orc.mask_dense(items, 70)
    assert bits.shape == (3,)
    assert set(orc.dense_to_tokens(bits, 70).tolist()) == set(items[:, 0].tolist())
    for t in range(70, 96):
        assert (bits[t >> 5] >> (t & 31)) & 1 == 0


def test_csr_rows(orc):
    items = _random_items(11, 300, 3, 9)
    si = orc.SortedItems(items, 9)
    prefixes = np.array([items[0, :2], items[5, :2], [8, 8], items[7, :2]], np.int32)
    live = np.array([1, 1, 1, 0], np.uint8)
    row_ptr, cols = si.mask_csr(2, prefixes, live)
    assert row_ptr[0] == 0 and np.all(np.diff(row_ptr) >= 0)
    assert row_ptr[4] - row_ptr[3] == 0                 # dead row is empty
    for r in range(3):
        want = orc.next_tokens_scan(items, prefixes[r], 9)
        assert cols[row_ptr[r]:row_ptr[r + 1]].tolist() == want.tolist()

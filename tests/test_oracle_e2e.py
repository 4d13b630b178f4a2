"""End-to-end pins of the oracle's beam decode (CPU only).

Definitions pinned: xGR page 2.1 (token-granular Unshared cache, in-place
updates by direct indices) and 2.2 (valid-path masks, top-K beam search).

* With path-consistent scores and a beam at least as wide as the item set,
  nothing is ever pruned, so the final beams are exactly all items ranked by
  their total fp32 score: enumerate the items directly and compare.
* The ancestry rewired in place equals the walk back over the per-step parent
  arrays (a second formulation).
* Every emitted sequence is a valid item; cum is the fp32 left fold of the
  log-probs along the path.
"""
import hashlib

import numpy as np
import pytest

import workloads


def _lp(path, t):
    """Deterministic, path-consistent log-prob in [-6, 0) on a coarse grid (ties happen)."""
    h = hashlib.blake2b(repr((tuple(path), t)).encode(), digest_size=4).digest()
    return np.float32(-(int.from_bytes(h, "little") % 48) / 8.0)


def _scores(dec, s, V):
    lp = np.full((dec.BW, V), -100.0, np.float32)
    for b in range(dec.n_live):
        path = dec.paths[b, :s].tolist()
        for t in range(V):
            lp[b, t] = _lp(path, t)
    return lp


def _run(orc, items, V, BW, K, S, method=0, n_heads=(2, 1), D=8, P=5, seed=0):
    si = orc.SortedItems(items, V)
    Hq, Hkv = n_heads
    dec = orc.BeamDecode(si, BW, K, S, Hq, Hkv, D, V, mode="logprob")
    rng = np.random.default_rng(seed)
    ks = rng.integers(0, 2 ** 16, size=(Hkv, P, D), dtype=np.uint16) & 0x3FFF
    vs = ks.copy()
    dec.begin(ks, vs)
    history = []
    for s in range(S):
        q = (rng.integers(0, 2 ** 16, size=(BW, Hq, D), dtype=np.uint16) & 0x3FFF)
        kn = (rng.integers(0, 2 ** 16, size=(BW, Hkv, D), dtype=np.uint16) & 0x3FFF)
        dec.attention(s, q, kn, kn)
        mask = dec.mask(s)
        lp = _scores(dec, s, V)
        history.append(lp)
        dec.select(s, lp, mask, method=method)
    return dec, history


@pytest.mark.parametrize("method", [0, 1, 2])
def test_wide_beam_returns_all_items_ranked(orc, method):
    V, L = 6, 3
    rng = np.random.default_rng(3)
    codes = rng.choice(V ** L, size=40, replace=False)
    items = np.stack([codes // 36, (codes // 6) % 6, codes % 6], 1).astype(np.int32)
    dec, _ = _run(orc, items, V, BW=48, K=48, S=L, method=method)
    ranked = []
    for it in items.tolist():
        c = np.float32(0.0)
        for s in range(L):
            c = np.float32(c + _lp(it[:s], it[s]))
        ranked.append((-float(c), it, c))
    # ties between items: the decode orders them by parent slot, i.e. by the
    # rank of their prefixes, so compare the multiset of (score, item) and the
    # non-increasing order rather than a particular tie order.
    ranked.sort(key=lambda x: x[0])
    assert dec.n_live == len(items)
    got = [(float(dec.cum[b]), tuple(dec.paths[b])) for b in range(dec.n_live)]
    assert sorted(got) == sorted((float(c), tuple(it)) for _, it, c in ranked)
    assert all(got[i][0] >= got[i + 1][0] for i in range(len(got) - 1))
    assert np.all(dec.paths[dec.n_live:] == -1)


def test_ancestry_two_formulations_agree(orc):
    w = workloads.WORKLOADS[1]
    items = workloads.items(w)
    dec, _ = _run(orc, items, w.V, BW=4, K=4, S=3)
    # after the last step anc holds slots of steps 0..S-1 for the final beams
    for b in range(dec.n_live):
        back = orc.ancestry_backward(dec.parents, 3, b)
        assert dec.anc[b, :3].tolist() == back[:3]
    # and mid-decode, for every live beam of every step
    dec2, _ = _run(orc, items, w.V, BW=4, K=4, S=3, seed=1)
    for b in range(dec2.n_live):
        assert all(0 <= x < 4 for x in dec2.anc[b, :3])


def test_sequences_valid_and_cum_is_fp32_fold(orc):
    w = workloads.WORKLOADS[1]
    items = workloads.items(w)
    item_set = {tuple(x) for x in items.tolist()}
    dec, hist = _run(orc, items, w.V, BW=4, K=4, S=3, seed=2)
    assert dec.n_live == 4
    for b in range(dec.n_live):
        path = tuple(dec.paths[b].tolist())
        assert path in item_set
        # recompute the fold along the path with the beam slots of each step
        c = np.float32(0.0)
        x = b
        slots = orc.ancestry_backward(dec.parents, 3, b)
        for s in range(3):
            c = np.float32(c + hist[s][slots[s], path[s]])
        assert c.tobytes() == np.float32(dec.cum[b]).tobytes()


def test_rewire_matches_parent_rows(orc):
    """In-place rewiring: beam b' of step s+1 owns slot b' at step s+1 and its
    parent's slots before that."""
    anc = np.array([[0, 0, -1], [1, 1, -1], [2, 0, -1]], np.int32)
    parent = np.array([2, 2, 0], np.int32)
    new = orc.ancestry_forward(anc, parent, 2, 3)
    assert new.tolist() == [[2, 0, 0], [2, 0, 1], [0, 0, 2]]
    new = orc.ancestry_forward(anc, parent, 2, 2)
    assert new.tolist() == [[2, 0, 0], [2, 0, 1], [-1, -1, -1]]

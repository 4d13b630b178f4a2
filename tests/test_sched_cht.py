"""The host-side batch former (Chunked Hash Tree, include/xgr_sched.h) against
its oracle (oracle/batching.py, token comparisons, no hashing), and the oracle
against a hand-derived example.  CPU only."""
import numpy as np
import pytest

from oracle.batching import BatchFormerOracle
from shared_prefix_decode_xattention_b200 import build, xgr
from shared_prefix_decode_xattention_b200.sched import ChunkedHashTree

import workloads


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


# Chunks of 2 tokens.  A = [1 2|3 4|5 6], B = [1 2|3 4|7 8], C = [9 9|1 2],
# D = [1 2|3 4|5 6|7] (3 full chunks), E = [1 2|8 8], F = [1 2|3 4|7 8|9 9],
# inserted A..F.  Shared leading chunks: A-B 2, A-D 3, A-E 1, A-F 2, B-D 2,
# B-E 1, B-F 3, D-E 1, D-F 2, E-F 1, C-anything 0.
# max_batch 10, min_shared 1: A seeds (tip 3).  Missing: B 1, C 2, D 0, E 1,
# F 2 -> D (depth 3).  B (1, older than E; depth 2, tip 2).  Now E 1 and F 1
# (F's coverage comes from B, 3 chunks) -> E, older (depth min(2, 1) = 1).
# Then F 1 against C 2 -> F (depth min(1, 2) = 1).  C would leave depth 0:
# dispatch [A D B E F] sharing 1; then C alone (its own 2 chunks).
# min_shared 2: A, D, B as before (tip 2); E (missing 1) would leave depth 1 < 2
# and is passed over; F (missing 1, younger) keeps depth 2: [A D B F] sharing 2.
# C seeds; E (missing 2) would leave depth 0: [C] 2.  E seeds alone: [E] 2.
HAND = {"A": [1, 2, 3, 4, 5, 6], "B": [1, 2, 3, 4, 7, 8], "C": [9, 9, 1, 2],
        "D": [1, 2, 3, 4, 5, 6, 7], "E": [1, 2, 8, 8], "F": [1, 2, 3, 4, 7, 8, 9, 9]}
IDS = {k: i + 1 for i, k in enumerate("ABCDEF")}
HAND_EXPECT = {
    1: [(["A", "D", "B", "E", "F"], 1), (["C"], 2)],
    2: [(["A", "D", "B", "F"], 2), (["C"], 2), (["E"], 2)],
}


def _named(batches):
    inv = {v: k for k, v in IDS.items()}
    return [([inv[i] for i in ids], sh) for ids, sh in batches]


@pytest.mark.parametrize("min_shared", [1, 2])
def test_oracle_hand_example(min_shared):
    o = BatchFormerOracle(2)
    for k in "ABCDEF":
        o.insert(IDS[k], HAND[k])
    assert _named(o.form_batches(10, min_shared)) == HAND_EXPECT[min_shared]


@pytest.mark.parametrize("min_shared", [1, 2])
def test_tree_hand_example(min_shared):
    t = ChunkedHashTree(2)
    for k in "ABCDEF":
        t.insert(IDS[k], HAND[k])
    assert _named(t.form_batches(10, min_shared)) == HAND_EXPECT[min_shared]


def test_hand_example_step_by_step():
    """find_best's (missing, depth_after, delta, w) on the example, both sides."""
    o, t = BatchFormerOracle(2), ChunkedHashTree(2)
    for k in "ABCDEF":
        o.insert(IDS[k], HAND[k])
        t.insert(IDS[k], HAND[k])
    # empty batch: the oldest (A) seeds; it keeps its 3 chunks; D also holds
    # A's third chunk, so w = 1
    assert o.find_best() == t.find_best() == (IDS["A"], 3, 3, 0, 1)
    for side in (o, t):
        side.add(IDS["A"])
    # D: missing 0, depth 3, delta 0; nobody else shares 3 chunks with D
    assert o.find_best() == t.find_best() == (IDS["D"], 0, 3, 0, 0)
    for side in (o, t):
        side.add(IDS["D"])
    # B: missing 1, depth 2 (delta 1); of the waiting requests F shares B's
    # first 2 chunks, so w = 1
    assert o.find_best() == t.find_best() == (IDS["B"], 1, 2, 1, 1)


# A request sharing nothing with the batch (Z: shorter than a chunk, so it
# misses no chunk at all) arrives between requests that share A's whole
# prompt.  Chunks of 4; A = 32 tokens (8 chunks), Z = 2 tokens (0 chunks),
# B and C = A's tokens + 8 of their own (10 chunks); inserted A, Z, B, C;
# max_batch 16, min_shared 1.  A seeds (tip 8).  Z ranks first by missing
# count (0) but would leave depth 0 < 1: passed over.  B (missing 2, depth 8,
# older than C) joins, then C (missing 2: its first 8 chunks are covered).
# Only Z is left and it fails the floor: dispatch [A B C] sharing 8, then [Z]
# sharing 0 (it has no full chunk).
SHORT = {"A": list(range(32)), "Z": [100, 101], "B": list(range(32)) + list(range(40, 48)),
         "C": list(range(32)) + list(range(50, 58))}
SHORT_IDS = {"A": 10, "Z": 11, "B": 12, "C": 13}
SHORT_EXPECT = [(["A", "B", "C"], 8), (["Z"], 0)]


# Coverage counts the member sharing the MOST with a candidate.  Chunks of 1;
# P = [1 2 3], Q = [1 2 9], X = [1 2 3 4], W = [1 5], inserted P, Q, X, W;
# max_batch 10, min_shared 1.  P seeds (tip 3): Q, X and W all miss one chunk
# -> Q, the oldest (tip 2).  X now misses 4 - max(3 with P, 2 with Q) = 1 and
# W misses 1: X, older, joins (depth 2), then W (depth 1).  [P Q X W] sharing 1.
MAXCOV = {"P": [1, 2, 3], "Q": [1, 2, 9], "X": [1, 2, 3, 4], "W": [1, 5]}
MAXCOV_IDS = {"P": 20, "Q": 21, "X": 22, "W": 23}
MAXCOV_EXPECT = [(["P", "Q", "X", "W"], 1)]


def _maxcov_named(batches):
    inv = {v: k for k, v in MAXCOV_IDS.items()}
    return [([inv[i] for i in ids], sh) for ids, sh in batches]


def test_coverage_by_the_most_sharing_member():
    for side in (BatchFormerOracle(1), ChunkedHashTree(1)):
        for k in "PQXW":
            side.insert(MAXCOV_IDS[k], MAXCOV[k])
        assert _maxcov_named(side.form_batches(10, 1)) == MAXCOV_EXPECT, type(side).__name__


def _short_named(batches):
    inv = {v: k for k, v in SHORT_IDS.items()}
    return [([inv[i] for i in ids], sh) for ids, sh in batches]


def test_short_prompt_does_not_end_a_batch():
    for side in (BatchFormerOracle(4), ChunkedHashTree(4)):
        for k in "AZBC":
            side.insert(SHORT_IDS[k], SHORT[k])
        assert _short_named(side.form_batches(16, 1)) == SHORT_EXPECT, type(side).__name__


def test_negative_request_id_is_rejected():
    t = ChunkedHashTree(2)
    with pytest.raises(xgr.XgrError) as e:
        t.insert(-1, [1, 2, 3])
    assert e.value.status == xgr.XGR_ERR_ARG


def _family_workload(rng, n_req, n_fam, chunk, vocab=50):
    """Requests from a few prompt families: a family prefix, then a private
    random tail; some share longer sub-prefixes, some are shorter than a chunk."""
    fams = [rng.integers(0, vocab, size=int(rng.integers(0, 6 * chunk + 1))) for _ in range(n_fam)]
    reqs = []
    for _ in range(n_req):
        f = fams[int(rng.integers(0, n_fam))]
        cut = int(rng.integers(0, len(f) + 1)) if rng.random() < 0.3 else len(f)
        tail = rng.integers(0, vocab, size=int(rng.integers(0, 4 * chunk + 1)))
        reqs.append(np.concatenate([f[:cut], tail]).astype(np.int32))
    return reqs


@pytest.mark.parametrize("seed", range(12))
def test_tree_matches_oracle_on_random_families(seed):
    rng = np.random.default_rng(1000 + seed)
    chunk = [1, 2, 3, 8][seed % 4]
    reqs = _family_workload(rng, int(rng.integers(1, 60)), int(rng.integers(1, 6)), chunk)
    max_batch = [1, 3, 8, 1000][seed % 4]
    min_shared = [0, 1, 2][seed % 3]
    o, t = BatchFormerOracle(chunk), ChunkedHashTree(chunk)
    ids = rng.permutation(10_000)[:len(reqs)]   # arbitrary non-negative ids
    for i, r in zip(ids, reqs):
        o.insert(int(i), r)
        t.insert(int(i), r)
    assert t.form_batches(max_batch, min_shared) == o.form_batches(max_batch, min_shared)
    assert t.counts() == (0, 0)


@pytest.mark.parametrize("seed", range(8))
def test_incremental_operations_match_oracle(seed):
    """Random interleavings of insert / remove / find_best / add / dispatch."""
    rng = np.random.default_rng(2000 + seed)
    chunk = [1, 4][seed % 2]
    pool = _family_workload(rng, 80, 4, chunk)
    o, t = BatchFormerOracle(chunk), ChunkedHashTree(chunk)
    next_id, waiting = 0, []
    for _ in range(300):
        op = rng.random()
        if op < 0.35 or not waiting:
            r = pool[int(rng.integers(0, len(pool)))]
            o.insert(next_id, r)
            t.insert(next_id, r)
            waiting.append(next_id)
            next_id += 1
        elif op < 0.45:
            victim = waiting[int(rng.integers(0, len(waiting)))]
            o.remove(victim)
            t.remove(victim)
            waiting.remove(victim)
        elif op < 0.85:
            b = o.find_best()
            assert t.find_best() == b
            if b is not None and rng.random() < 0.8:
                o.add(b[0])
                t.add(b[0])
                waiting.remove(b[0])
        else:
            assert t.dispatch() == o.dispatch()
        assert t.counts() == (len(o.waiting), len(o.batch))


def test_groups_of_the_prefix_shared_llm_workload():
    """Workload 4's batch: 64 requests in 4 groups sharing 8192-token prefixes,
    each with a private 256..2048-token suffix, arriving interleaved.  With
    256-token chunks the tree forms exactly the 4 groups, each sharing its 32
    prefix chunks."""
    w = workloads.WORKLOADS[4]
    rng = np.random.default_rng(7)
    prefixes = [rng.integers(0, 32000, size=w.prompt[0]) for _ in range(w.groups)]
    suf = workloads.suffix_lengths(w)
    t = ChunkedHashTree(256)
    order = rng.permutation(w.B)
    for r in order:
        tail = rng.integers(0, 32000, size=int(suf[r]))
        t.insert(int(r), np.concatenate([prefixes[w.shared_id(int(r))], tail]).astype(np.int32))
    batches = t.form_batches(max_batch=w.B, min_shared_chunks=16)
    assert len(batches) == w.groups
    for ids, sh in batches:
        assert sh == w.prompt[0] // 256
        assert len({w.shared_id(i) for i in ids}) == 1 and len(ids) == w.B // w.groups


def test_errors_and_states():
    t = ChunkedHashTree(4)
    t.insert(1, [1, 2, 3, 4])
    with pytest.raises(xgr.XgrError) as e:
        t.insert(1, [5, 6, 7, 8])                # duplicate live id
    assert e.value.status == xgr.XGR_ERR_ARG
    t.add(1)
    with pytest.raises(xgr.XgrError) as e:
        t.remove(1)                              # a member of the batch being formed
    assert e.value.status == xgr.XGR_ERR_STATE
    with pytest.raises(xgr.XgrError) as e:
        t.add(1)
    assert e.value.status == xgr.XGR_ERR_STATE
    with pytest.raises(xgr.XgrError) as e:
        t.remove(99)                             # unknown id
    assert e.value.status == xgr.XGR_ERR_ARG
    assert t.dispatch() == ([1], 1)
    t.insert(1, [1, 2, 3, 4])                    # the id is free again after dispatch
    assert t.find_best() == (1, 1, 1, 0, 0)
    with pytest.raises(xgr.XgrError) as e:
        ChunkedHashTree(0)
    assert e.value.status == xgr.XGR_ERR_SHAPE


def test_long_running_tree_compacts_and_stays_exact():
    """Sixty rounds of 50 requests through one tree (3000 departures: the
    tables are compacted several times); every round's batches match the
    oracle's, with ids reused across rounds."""
    rng = np.random.default_rng(99)
    t = ChunkedHashTree(4)
    for rnd in range(60):
        reqs = _family_workload(rng, 50, 3, 4)
        o = BatchFormerOracle(4)
        for i, r in enumerate(reqs):
            o.insert(i, r)
            t.insert(i, r)
        assert t.form_batches(6, 1) == o.form_batches(6, 1), f"round {rnd}"


def _hand_outcomes(oracle_cls):
    """Everything the hand examples pin: both formations, the short-prompt
    formation and the step-by-step find_best values."""
    res = []
    o = oracle_cls(4)
    for k in "AZBC":
        o.insert(SHORT_IDS[k], SHORT[k])
    res.append(_short_named(o.form_batches(16, 1)))
    o = oracle_cls(1)
    for k in "PQXW":
        o.insert(MAXCOV_IDS[k], MAXCOV[k])
    res.append(_maxcov_named(o.form_batches(10, 1)))
    for ms in (1, 2):
        o = oracle_cls(2)
        for k in "ABCDEF":
            o.insert(IDS[k], HAND[k])
        res.append(_named(o.form_batches(10, ms)))
    o = oracle_cls(2)
    for k in "ABCDEF":
        o.insert(IDS[k], HAND[k])
    steps = [o.find_best()]
    o.add(IDS["A"])
    steps.append(o.find_best())
    o.add(IDS["D"])
    steps.append(o.find_best())
    return res, steps


def _mutant(name):
    """A copy of the oracle with one plausible mistake planted."""
    class M(BatchFormerOracle):
        pass
    if name == "newest first on ties":
        def find_best(self):
            w0 = list(self.waiting)
            self.waiting = w0[::-1]
            try:
                return BatchFormerOracle.find_best(self)
            finally:
                self.waiting = w0
        M.find_best = find_best
    elif name == "coverage by the least-sharing member":
        M.missing = lambda self, r: (self.chunks(r) if not self.batch
                                     else self.chunks(r) - min(self.shared(r, m) for m in self.batch))
    elif name == "tip as the deepest member":
        M.tip = lambda self: (0 if not self.batch else
                              max(self.shared(m, self.batch[0]) if m != self.batch[0]
                                  else self.chunks(m) for m in self.batch))
    elif name == "dispatch when the best request fails the floor":
        def form_batches(self, max_batch, min_shared_chunks):
            res = []
            while self.waiting:
                self.add(self.find_best()[0])
                while len(self.batch) < max_batch:
                    best = self.find_best()
                    if best is None or best[2] < min_shared_chunks:
                        break
                    self.add(best[0])
                res.append(self.dispatch())
            return res
        M.form_batches = form_batches
    elif name == "stop at equality":
        def form_batches(self, max_batch, min_shared_chunks):
            return BatchFormerOracle.form_batches(self, max_batch, min_shared_chunks + 1)
        M.form_batches = form_batches
    elif name == "partial chunk counted":
        M.chunks = lambda self, r: -(-len(self.tokens[r]) // self.C)
    elif name == "w counts the candidate":
        def find_best(self):
            b = BatchFormerOracle.find_best(self)
            return None if b is None else b[:4] + (b[4] + (1 if b[2] > 0 else 0),)
        M.find_best = find_best
    return M


@pytest.mark.parametrize("name", ["newest first on ties", "coverage by the least-sharing member",
                                  "dispatch when the best request fails the floor",
                                  "tip as the deepest member", "stop at equality",
                                  "partial chunk counted", "w counts the candidate"])
def test_planted_mistakes_fail_the_hand_pins(name):
    good = ([SHORT_EXPECT, MAXCOV_EXPECT, HAND_EXPECT[1], HAND_EXPECT[2]],
            [(IDS["A"], 3, 3, 0, 1), (IDS["D"], 0, 3, 0, 0), (IDS["B"], 1, 2, 1, 1)])
    assert _hand_outcomes(BatchFormerOracle) == good
    assert _hand_outcomes(_mutant(name)) != good, name

"""Pins of the oracle's beam selection (CPU only).

Definition pinned: xGR page, 2.2 xBeam, "Early sort termination" -- the top
sequences of the candidate pool by cumulative log-probability, found with a
global min-heap that stops a branch at its first log-prob below the heap
minimum.  Readings: score = fp32(cum[b] + lp[b][t]); order = higher score, then
lower parent, then lower token; dead slots -1/-1/-inf; NaN is an error.
"""
import itertools
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f(x):
    return np.float32(float(x))


def _csr(valid):
    row_ptr = np.zeros(len(valid) + 1, np.int64)
    row_ptr[1:] = np.cumsum([len(v) for v in valid])
    cols = np.array([t for v in valid for t in v], np.int32)
    return row_ptr, cols


@pytest.mark.parametrize("method", [0, 1, 2])
def test_golden_cases(orc, method):
    fx = json.load(open(os.path.join(GOLDEN, "select_tiny.json")))
    for case in fx["cases"]:
        cum = np.array([_f(x) for x in case["cum"]], np.float32)
        lp = np.array([[_f(x) for x in row] for row in case["lp"]], np.float32)
        row_ptr, cols = _csr(case["valid"])
        parent, token, cum_out, n = orc.select_logprob(cum, lp, row_ptr, cols, case["BW"],
                                                       case["K"], case["n_live"], method)
        assert n == case["n_out"]
        assert parent.tolist() == case["parent"]
        assert token.tolist() == case["token"]
        want = np.array([_f(x) for x in case["cum_out"]], np.float32)
        assert want.tobytes() == cum_out.tobytes()      # bit-exact, +0.0 included


def _brute(cum, lp, valid, BW, n_live):
    """itertools over every (beam, token) pair, Python's sort on the total order."""
    cands = []
    for b, t in itertools.product(range(n_live), range(lp.shape[1])):
        if t in valid[b]:
            k = np.float32(cum[b]) + np.float32(lp[b, t])
            k = np.float32(0.0) if k == 0 else k
            cands.append((-float(k), b, t, k))
    cands.sort(key=lambda c: c[:3])
    return cands[:BW]


def _random_case(rng, n_live, V, BW, ties):
    cum = rng.normal(0, 2, size=BW).astype(np.float32)
    if ties:
        lp = (np.round(rng.normal(-3, 2, size=(BW, V)) * 2) / 2).astype(np.float32)
        cum = (np.round(cum * 2) / 2).astype(np.float32)
    else:
        lp = rng.normal(-3, 2, size=(BW, V)).astype(np.float32)
    lp[rng.random(lp.shape) < 0.03] = -np.inf
    valid = [sorted(rng.choice(V, size=rng.integers(0, V + 1), replace=False).tolist())
             for _ in range(BW)]
    return cum, lp, valid


@pytest.mark.parametrize("seed", range(12))
def test_three_algorithms_equal_brute_force(orc, seed):
    rng = np.random.default_rng(seed)
    BW = int(rng.integers(1, 9))
    V = int(rng.integers(1, 12))
    n_live = int(rng.integers(1, BW + 1))
    cum, lp, valid = _random_case(rng, n_live, V, BW, ties=seed % 2 == 0)
    row_ptr, cols = _csr(valid[:n_live] + [[]] * (BW - n_live))
    want = _brute(cum, lp, valid, BW, n_live)
    for method in (0, 1, 2):
        K = BW + int(rng.integers(0, 3))
        parent, token, cum_out, n = orc.select_logprob(cum, lp, row_ptr, cols, BW, K, n_live,
                                                       method)
        assert n == len(want)
        assert parent[:n].tolist() == [c[1] for c in want]
        assert token[:n].tolist() == [c[2] for c in want]
        assert cum_out[:n].tobytes() == np.array([c[3] for c in want], np.float32).tobytes()
        assert np.all(parent[n:] == -1) and np.all(token[n:] == -1)
        assert np.all(np.isneginf(cum_out[n:]))


def test_larger_pool_methods_agree(orc):
    rng = np.random.default_rng(77)
    BW, V = 64, 300
    cum, lp, valid = _random_case(rng, BW, V, BW, ties=True)
    row_ptr, cols = _csr(valid)
    outs = [orc.select_logprob(cum, lp, row_ptr, cols, BW, BW, BW, m) for m in (0, 1, 2)]
    for o in outs[1:]:
        for a, b in zip(outs[0][:3], o[:3]):
            assert a.tobytes() == b.tobytes()
    # invariants: non-increasing scores; candidates counted right
    c = outs[0][2]
    assert np.all(c[:-1] >= c[1:])
    assert outs[0][3] == min(BW, len(cols))


def test_two_stage_truncation_can_matter_only_when_K_below_BW(orc):
    """Per-beam top-K is a pure optimisation when K >= BW (the reading used);
    with K < BW a beam holding many winners is cut, which the flat sort is not."""
    cum = np.array([0.0, -10.0], np.float32)
    lp = np.array([[-1, -1.5, -2, -2.5], [-1, -1, -1, -1]], np.float32)
    row_ptr, cols = _csr([[0, 1, 2, 3], [0, 1, 2, 3]])
    flat = orc.select_logprob(cum, lp, row_ptr, cols, 4, 4, 2, 0)
    two = orc.select_logprob(cum, lp, row_ptr, cols, 4, 2, 2, 1)
    assert flat[0].tolist() == [0, 0, 0, 0]
    assert two[0].tolist() == [0, 0, 1, 1]


def test_nan_is_an_error(orc):
    cum = np.zeros(2, np.float32)
    lp = np.zeros((2, 3), np.float32)
    lp[1, 2] = np.nan
    row_ptr, cols = _csr([[0], [1, 2]])
    with pytest.raises(RuntimeError):
        orc.select_logprob(cum, lp, row_ptr, cols, 2, 2, 2, 0)
    # a NaN outside the valid set is never read
    row_ptr, cols = _csr([[0], [1]])
    orc.select_logprob(cum, lp, row_ptr, cols, 2, 2, 2, 0)


def test_logits_mode_matches_fp64_definition(orc):
    rng = np.random.default_rng(5)
    BW, V = 5, 40
    logits = rng.normal(0, 2, size=(BW, V)).astype(np.float32)
    cum = rng.normal(-3, 1, size=BW)
    valid = [sorted(rng.choice(V, size=int(rng.integers(1, V)), replace=False).tolist())
             for _ in range(BW)]
    row_ptr, cols = _csr(valid)
    parent, token, cum_out, n, lse = orc.select_logits(cum, logits, row_ptr, cols, BW, BW)
    x = logits.astype(np.float64)
    want_lse = np.log(np.exp(x).sum(-1))                    # no max shift needed at this scale
    assert np.allclose(lse, want_lse, atol=1e-12)
    cands = sorted(((-(cum[b] + x[b, t] - want_lse[b]), b, t) for b in range(BW)
                    for t in valid[b]))[:BW]
    assert parent.tolist() == [c[1] for c in cands]
    assert token.tolist() == [c[2] for c in cands]
    assert np.allclose(cum_out, [-c[0] for c in cands], atol=1e-12)

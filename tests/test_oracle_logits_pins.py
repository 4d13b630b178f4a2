"""Pins of the oracle's logits-mode selection (CPU only).

Definition pinned: xGR page, 2.2 xBeam, "Valid-path constraint" and "Early
sort termination".  Reading: a token's log-prob is its logit minus the
log-sum-exp of the whole row (masking after normalisation); the score is the
fp64 sum of the beam's cumulative score and that log-prob; ties go to the lower
parent, then the lower token.

The expected values (tests/golden/select_logits_tiny.json) are closed forms
worked by hand.  A second test plants plausible mistakes in a copy of the
oracle's C source -- normalising over the valid tokens only, no max shift in
the log-sum-exp, the score added in fp32, token compared before parent -- and
checks that every one of them fails at least one pin.
"""
import ctypes
import json
import math
import os
import subprocess

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "select_logits_tiny.json")


def _cases():
    return json.load(open(GOLDEN))["cases"]


def _csr(valid):
    row_ptr = np.zeros(len(valid) + 1, np.int64)
    row_ptr[1:] = np.cumsum([len(v) for v in valid])
    cols = np.array([t for v in valid for t in v], np.int32)
    return row_ptr, cols


def _num(x):
    return -math.inf if x == "-inf" else float(x)


def _check(case, parent, token, cum_out, n, lse):
    """True when every output matches the hand-worked case."""
    tol = case["tol"]
    if n != case["n_out"] or parent.tolist() != case["parent"] or token.tolist() != case["token"]:
        return False
    for got, want in zip(cum_out.tolist(), case["cum_out"]["value"]):
        want = _num(want)
        if math.isinf(want):
            if not (math.isinf(got) and got < 0):
                return False
        elif not (math.isfinite(got) and abs(got - want) <= tol):
            return False
    for got, want in zip(np.asarray(lse).tolist(), case["lse"]["value"]):
        if not (math.isfinite(got) and abs(got - _num(want)) <= tol):
            return False
    return True


def _inputs(case):
    V, BW, n_live = case["V"], case["BW"], case["n_live"]
    cum = np.zeros(BW, np.float64)
    cum[:n_live] = case["cum"]
    logits = np.zeros((BW, V), np.float32)
    logits[:n_live] = np.array(case["logits"], np.float32)
    row_ptr, cols = _csr(case["valid"])
    return V, BW, n_live, cum, logits, row_ptr, cols


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"][:40])
def test_hand_worked_cases(case):
    V, BW, n_live, cum, logits, row_ptr, cols = _inputs(case)
    parent, token, cum_out, n, lse = oracle.select_logits(cum, logits, row_ptr, cols, BW, n_live)
    assert _check(case, parent, token, cum_out, n, lse), case["name"]


def test_constant_row_is_minus_ln_v_exactly():
    """Any constant row: lp = -ln V to fp64 rounding, whatever the constant."""
    for V, c in ((1, 7.0), (5, -3.25), (8192, 0.0), (16384, 12.5)):
        logits = np.full((1, V), c, np.float32)
        row_ptr, cols = _csr([[V - 1]])
        _, _, cum_out, n, lse = oracle.select_logits(np.zeros(1), logits, row_ptr, cols, 1, 1)
        assert n == 1
        assert abs(cum_out[0] + math.log(V)) <= 1e-12 * max(1.0, math.log(V))
        assert abs(lse[0] - (c + math.log(V))) <= 1e-12 * max(1.0, abs(c) + math.log(V))


# ---------------------------------------------------------------- planted mistakes

_SRC = os.path.join(os.path.dirname(oracle.__file__), "xgr_oracle.c")

# (old text, new text) of the oracle's orc_select_logits / cmp64, per mistake
MISTAKES = {
    "normalised over the valid tokens only": [(
        "        double lse = m + log(l);",
        "        double lse; { double mv = -INFINITY, lv = 0.0;\n"
        "          for (int64_t e = row_ptr[b]; e < row_ptr[b + 1]; ++e) if (x[cols[e]] > mv) mv = x[cols[e]];\n"
        "          for (int64_t e = row_ptr[b]; e < row_ptr[b + 1]; ++e) lv += exp((double)x[cols[e]] - mv);\n"
        "          lse = mv + log(lv); (void)l; }")],
    "no max shift in the log-sum-exp": [
        ("        for (int t = 0; t < V; ++t) l += exp((double)x[t] - m);",
         "        for (int t = 0; t < V; ++t) l += exp((double)x[t]);"),
        ("        double lse = m + log(l);", "        double lse = log(l);")],
    "score added in fp32": [(
        "            all[c].key = cum[b] + ((double)x[t] - lse);",
        "            all[c].key = (double)((float)cum[b] + (float)((double)x[t] - lse));")],
    "token compared before parent": [(
        "    if (x->b != y->b) return x->b < y->b ? -1 : 1;\n"
        "    if (x->t != y->t) return x->t < y->t ? -1 : 1;\n"
        "    return 0;\n"
        "}\n"
        "\n"
        "/* The fp32 score",
        "    if (x->t != y->t) return x->t < y->t ? -1 : 1;\n"
        "    if (x->b != y->b) return x->b < y->b ? -1 : 1;\n"
        "    return 0;\n"
        "}\n"
        "\n"
        "/* The fp32 score")],
}


def _build_mutant(tmp_path, name):
    src = open(_SRC).read()
    for old, new in MISTAKES[name]:
        assert src.count(old) == 1, f"planting '{name}': the oracle text it replaces has changed"
        src = src.replace(old, new)
    c = tmp_path / "mutant.c"
    so = tmp_path / "libmutant.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                           "-ffp-contract=off", "-o", str(so), str(c), "-lm"])
    L = ctypes.CDLL(str(so))
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    L.orc_select_logits.argtypes = [i32, i32, i32, P, P, P, P, P, P, P, P]
    return L


def _run_raw(L, case):
    V, BW, n_live, cum, logits, row_ptr, cols = _inputs(case)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    parent = np.zeros(BW, np.int32)
    token = np.zeros(BW, np.int32)
    cum_out = np.zeros(BW, np.float64)
    lse = np.zeros(max(n_live, 1), np.float64)
    with np.errstate(all="ignore"):
        n = L.orc_select_logits(BW, V, n_live, p(cum), p(logits), p(row_ptr), p(cols), p(parent),
                                p(token), p(cum_out), p(lse))
    return parent, token, cum_out, n, lse[:n_live]


@pytest.mark.parametrize("name", list(MISTAKES))
def test_planted_mistakes_fail_a_pin(tmp_path, name):
    L = _build_mutant(tmp_path, name)
    failed = [c["name"] for c in _cases() if not _check(c, *_run_raw(L, c))]
    assert failed, f"mistake '{name}' passes every hand-worked case"


def test_unplanted_copy_passes(tmp_path):
    """The same build of an unmodified copy passes every case (the harness of the
    planted-mistake test is sound)."""
    MISTAKES["(none)"] = []
    try:
        L = _build_mutant(tmp_path, "(none)")
    finally:
        del MISTAKES["(none)"]
    for c in _cases():
        assert _check(c, *_run_raw(L, c)), c["name"]

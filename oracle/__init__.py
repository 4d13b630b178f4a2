"""CPU oracle for the xGR beam-decode hot path -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  It shares
no code with the CUDA library (``shared_prefix_decode_xattention_b200``) and
never imports it.

The arithmetic lives in ``xgr_oracle.c`` (plain loops, fp64, OpenMP over
independent rows); this module marshals numpy arrays into it and keeps the
per-request beam state (paths, ancestry, cumulative scores) in plain Python.

Sources: "xGR: Efficient Generative Recommendation Serving at Scale",
section 2.1 (xAttention: Shared prompt KV computed once, token-granular
Unshared KV, staged attention merged by online softmax, in-place updates by
direct indices) and section 2.2 (xBeam: valid-path masks from a pre-built item
vocabulary, early-terminating top-K with a global min-heap).

Parity status: every function below is pinned by tests/test_oracle_*.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "xgr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile xgr_oracle.c with gcc (fp64, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        L.orc_attend.argtypes = [i32, i32, P, i32, P, P, f64, P, P]
        L.orc_decode_attention.argtypes = [i32, i32, i32, i32, i32, i32, P, P, P, i32, P, P, i32,
                                           P, P, P, i32, P, i32, P, P]
        L.orc_next_tokens_scan.argtypes = [P, i64, i32, i32, P, i32, P]
        L.orc_sort_items.argtypes = [P, i64, i32]
        L.orc_sort_items.restype = None
        L.orc_next_tokens_sorted.argtypes = [P, i64, i32, P, i32, P]
        L.orc_mask_dense.argtypes = [P, i64, i32, i32, P]
        L.orc_mask_dense.restype = None
        L.orc_mask_csr.argtypes = [P, i64, i32, i32, i32, i32, P, i32, P, P, P, i64]
        L.orc_mask_csr.restype = i64
        L.orc_select_logprob.argtypes = [i32, i32, i32, i32, P, P, P, P, i32, P, P, P]
        L.orc_select_logits.argtypes = [i32, i32, i32, P, P, P, P, P, P, P, P]
        L.orc_num_threads.argtypes = []
        L.orc_set_num_threads.argtypes = [i32]
        L.orc_set_num_threads.restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """bf16 data as its raw uint16 bits (accepts a torch bf16 tensor or uint16 array)."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint16
        return np.ascontiguousarray(a)
    import torch
    t = a.detach().to("cpu").contiguous()
    assert t.dtype == torch.bfloat16
    return t.view(torch.int16).numpy().view(np.uint16)


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))


# ---------------------------------------------------------------- attention

def attend(q, k, v, scale: Optional[float] = None):
    """Plain softmax attention of q [n_q][D] over keys k, v [n][D] (bf16).
    Returns (out fp64 [n_q][D], lse fp64 [n_q])."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    n_q, D = q.shape
    n = k.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((n_q, D), np.float64)
    lse = np.zeros((n_q,), np.float64)
    rc = lib().orc_attend(n_q, D, _p(q), n, _p(k), _p(v), float(scale), _p(out), _p(lse))
    if rc:
        raise RuntimeError(f"orc_attend failed: {rc}")
    return out, lse


def decode_attention(q, ks, vs, kpool, vpool, anc, s: int, n_live: int, kx=None, vx=None,
                     beams=None):
    """Attention of one request at step s over shared prompt + optional suffix +
    the beams' own Unshared tokens (see xgr_oracle.c).

    q [BW][Hq][D]; ks, vs [Hkv][P][D]; kx, vx [Hkv][X][D] or None;
    kpool, vpool [S'][BW][Hkv][D] (S' > s); anc int32 [BW][>s].
    beams: optional list of beam ids to compute (q then holds only those rows).
    Returns out fp64 [n][Hq][D], lse fp64 [n][Hq] (n = BW or len(beams))."""
    q, ks, vs, kpool, vpool = _u16(q), _u16(ks), _u16(vs), _u16(kpool), _u16(vpool)
    BW = kpool.shape[1]
    _, Hq, D = q.shape
    Hkv, P, _ = ks.shape
    if kx is None:
        kx = np.zeros((Hkv, 0, D), np.uint16)
        vx = np.zeros((Hkv, 0, D), np.uint16)
    kx, vx = _u16(kx), _u16(vx)
    X = kx.shape[1]
    anc = np.ascontiguousarray(anc, dtype=np.int32)
    assert kpool.shape[1:] == (BW, Hkv, D) and kpool.shape[0] > s
    ids = None if beams is None else np.ascontiguousarray(beams, dtype=np.int32)
    n = BW if ids is None else len(ids)
    assert q.shape[0] == n
    out = np.zeros((n, Hq, D), np.float64)
    lse = np.zeros((n, Hq), np.float64)
    rc = lib().orc_decode_attention(BW, Hq, Hkv, D, s, n_live, _p(q), _p(ks), _p(vs), P,
                                    _p(kx), _p(vx), X, _p(kpool), _p(vpool), _p(anc),
                                    anc.shape[1], None if ids is None else _p(ids),
                                    0 if ids is None else n, _p(out), _p(lse))
    if rc:
        raise RuntimeError(f"orc_decode_attention failed: {rc}")
    return out, lse


# ---------------------------------------------------------------- masks

def next_tokens_scan(items: np.ndarray, prefix, V: int) -> np.ndarray:
    """Brute force: valid next tokens of ``prefix`` by scanning every item."""
    items = np.ascontiguousarray(items, dtype=np.int32)
    N, L = items.shape
    pre = np.ascontiguousarray(np.asarray(prefix, dtype=np.int32).reshape(-1))
    out = np.zeros((V,), np.int32)
    c = lib().orc_next_tokens_scan(_p(items), N, L, V, _p(pre) if pre.size else None,
                                   pre.size, _p(out))
    if c < 0:
        raise RuntimeError("scan failed")
    return out[:c].copy()


def mask_dense(items: np.ndarray, V: int) -> np.ndarray:
    """Dense first-step mask: uint32 [ceil(V/32)], bit t%32 of word t/32."""
    items = np.ascontiguousarray(items, dtype=np.int32)
    bits = np.zeros(((V + 31) // 32,), np.uint32)
    lib().orc_mask_dense(_p(items), items.shape[0], items.shape[1], V, _p(bits))
    return bits


def dense_to_tokens(bits: np.ndarray, V: int) -> np.ndarray:
    t = np.arange(V)
    return t[(bits[t >> 5] >> (t & 31).astype(np.uint32)) & 1 == 1].astype(np.int32)


class SortedItems:
    """The item vocabulary sorted lexicographically once; prefix ranges by binary search."""

    def __init__(self, items: np.ndarray, V: int):
        self.items = np.array(items, dtype=np.int32, copy=True, order="C")
        self.N, self.L = self.items.shape
        self.V = V
        lib().orc_sort_items(_p(self.items), self.N, self.L)

    def next_tokens(self, prefix) -> np.ndarray:
        pre = np.ascontiguousarray(np.asarray(prefix, dtype=np.int32).reshape(-1))
        out = np.zeros((self.V,), np.int32)
        c = lib().orc_next_tokens_sorted(_p(self.items), self.N, self.L,
                                         _p(pre) if pre.size else None, pre.size, _p(out))
        return out[:c].copy()

    def mask_csr(self, s: int, prefixes: np.ndarray, live: np.ndarray, cap: Optional[int] = None):
        """CSR rows (int64 row_ptr, int32 cols) of the valid next tokens of each
        row's prefix (prefixes int32 [n_rows][>=s]); dead rows are empty."""
        prefixes = np.ascontiguousarray(prefixes, dtype=np.int32)
        n_rows = prefixes.shape[0]
        live = np.ascontiguousarray(live, dtype=np.uint8)
        if cap is None:
            cap = n_rows * self.V
        row_ptr = np.zeros((n_rows + 1,), np.int64)
        cols = np.zeros((max(cap, 1),), np.int32)
        nnz = lib().orc_mask_csr(_p(self.items), self.N, self.L, self.V, s, n_rows, _p(prefixes),
                                 prefixes.shape[1], _p(live), _p(row_ptr), _p(cols), cap)
        if nnz < 0:
            raise RuntimeError("mask capacity too small")
        return row_ptr, cols[:nnz].copy()


# ---------------------------------------------------------------- selection

def select_logprob(cum, lp, row_ptr, cols, BW: int, K: int, n_live: int, method: int = 0):
    """Log-prob mode selection (fp32 scores, bit-exact contract).
    cum fp32 [>=n_live]; lp fp32 [>=n_live][V]; CSR rows per live beam.
    method 0 = flat sort, 1 = per-beam top-K then global, 2 = min-heap early termination.
    Returns parent, token (int32 [BW]), cum_out (fp32 [BW]), n_out."""
    cum = np.ascontiguousarray(cum, dtype=np.float32)
    lp = np.ascontiguousarray(lp, dtype=np.float32)
    V = lp.shape[-1]
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int32)
    parent = np.zeros((BW,), np.int32)
    token = np.zeros((BW,), np.int32)
    cum_out = np.zeros((BW,), np.float32)
    n = lib().orc_select_logprob(BW, K, V, n_live, _p(cum), _p(lp), _p(row_ptr),
                                 _p(cols) if cols.size else None, method,
                                 _p(parent), _p(token), _p(cum_out))
    if n < 0:
        raise RuntimeError(f"orc_select_logprob failed: {n}")
    return parent, token, cum_out, int(n)


def select_logits(cum, logits, row_ptr, cols, BW: int, n_live: int):
    """Logits mode selection, fp64 (normalise each row over the full vocabulary).
    Returns parent, token, cum_out (fp64), n_out, lse (fp64 [n_live])."""
    cum = np.ascontiguousarray(cum, dtype=np.float64)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    V = logits.shape[-1]
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int32)
    parent = np.zeros((BW,), np.int32)
    token = np.zeros((BW,), np.int32)
    cum_out = np.zeros((BW,), np.float64)
    lse = np.zeros((max(n_live, 1),), np.float64)
    n = lib().orc_select_logits(BW, V, n_live, _p(cum), _p(logits), _p(row_ptr),
                                _p(cols) if cols.size else None,
                                _p(parent), _p(token), _p(cum_out), _p(lse))
    if n < 0:
        raise RuntimeError(f"orc_select_logits failed: {n}")
    return parent, token, cum_out, int(n), lse[:n_live]


def logits_keys(cum, logits, pairs):
    """fp64 score of given (beam, token) pairs in logits mode (for tie-aware checks)."""
    logits = np.asarray(logits, dtype=np.float64)
    m = logits.max(axis=-1, keepdims=True)
    lse = (m + np.log(np.exp(logits - m).sum(axis=-1, keepdims=True)))[:, 0]
    return np.array([cum[b] + (logits[b, t] - lse[b]) for b, t in pairs], dtype=np.float64)


# ---------------------------------------------------------------- ancestry

def ancestry_forward(anc_prev: np.ndarray, parent: np.ndarray, s_next: int, n_out: int) -> np.ndarray:
    """Rewire after the selection of step s_next-1 (xGR 2.1 "In-place updates"):
    new beam b' inherits its parent's slots for steps < s_next and owns slot b'
    at step s_next.  Dead beams keep -1."""
    BW, S = anc_prev.shape
    anc = np.full_like(anc_prev, -1)
    for b in range(n_out):
        p = parent[b]
        for i in range(s_next):
            anc[b, i] = anc_prev[p, i]
        if s_next < S:
            anc[b, s_next] = b
    return anc


def ancestry_backward(parents: list, s: int, b: int) -> list:
    """Second formulation: walk the per-step parent arrays back from beam b of
    step s.  parents[j][x] = parent (a beam of step j) of beam x of step j+1."""
    out = [0] * (s + 1)
    x = b
    out[s] = x
    for j in range(s - 1, -1, -1):
        x = int(parents[j][x])
        out[j] = x
    return out


# ---------------------------------------------------------------- end to end

class BeamDecode:
    """Exhaustive beam search of one request, every step as the plain definitions.

    mode "logprob": fp32 scores/cum (bit-exact contract); "logits": fp64 scores.
    Each step returns attention output, the step's mask, and the selection.
    """

    def __init__(self, sorted_items: Optional[SortedItems], BW: int, K: int, S: int,
                 Hq: int, Hkv: int, D: int, V: int, mode: str = "logprob"):
        self.items = sorted_items
        self.BW, self.K, self.S, self.Hq, self.Hkv, self.D, self.V = BW, K, S, Hq, Hkv, D, V
        self.mode = mode

    def begin(self, ks, vs, kx=None, vx=None):
        BW, S = self.BW, self.S
        self.ks, self.vs, self.kx, self.vx = _u16(ks), _u16(vs), kx, vx
        self.n_live = 1
        self.cum = np.zeros((BW,), np.float32 if self.mode == "logprob" else np.float64)
        self.paths = np.full((BW, S), -1, np.int32)
        self.anc = np.full((BW, S), -1, np.int32)
        self.anc[0, 0] = 0
        self.parents = []
        self.kpool = np.zeros((S, BW, self.Hkv, self.D), np.uint16)
        self.vpool = np.zeros((S, BW, self.Hkv, self.D), np.uint16)

    def attention(self, s: int, q, k_new, v_new, beams=None):
        """Append this step's k/v at slot (s, b) of the Unshared pool, then attend
        (all beams, or only the listed ones)."""
        self.kpool[s] = _u16(k_new)
        self.vpool[s] = _u16(v_new)
        qq = _u16(q)
        if beams is not None:
            qq = np.ascontiguousarray(qq[np.asarray(beams)])
        return decode_attention(qq, self.ks, self.vs, self.kpool, self.vpool, self.anc, s,
                                self.n_live, self.kx, self.vx, beams=beams)

    def mask(self, s: int):
        """Step 0: dense bitset of valid first tokens.  Step >= 1: CSR rows over
        all BW beams (dead rows empty)."""
        if s == 0:
            return ("dense", mask_dense(self.items.items, self.V))
        live = (np.arange(self.BW) < self.n_live).astype(np.uint8)
        row_ptr, cols = self.items.mask_csr(s, self.paths, live)
        return ("csr", (row_ptr, cols))

    def _rows(self, s: int, mask):
        if s == 0:
            toks = dense_to_tokens(mask[1], self.V)
            row_ptr = np.zeros((self.BW + 1,), np.int64)
            row_ptr[1:] = len(toks)
            return row_ptr, toks
        return mask[1]

    def select(self, s: int, scores, mask, method: int = 0, force=None):
        """Select the next beams and rewire; ``force`` = (parent, token, n_out)
        replaces the choice (logits-mode teacher forcing after a tie-aware check)."""
        row_ptr, cols = self._rows(s, mask)
        scores = np.ascontiguousarray(scores, dtype=np.float32)
        if self.mode == "logprob":
            parent, token, cum, n = select_logprob(self.cum, scores, row_ptr, cols, self.BW,
                                                   self.K, self.n_live, method)
        else:
            parent, token, cum, n, _ = select_logits(self.cum, scores, row_ptr, cols,
                                                     self.BW, self.n_live)
            if force is not None:
                parent, token, n = (np.array(force[0], np.int32), np.array(force[1], np.int32),
                                    int(force[2]))
                pairs = [(int(parent[i]), int(token[i])) for i in range(n)]
                cum = np.full((self.BW,), -np.inf)
                cum[:n] = logits_keys(self.cum, scores, pairs)
        self._advance(s, parent, token, cum, n)
        return parent, token, cum, n

    def _advance(self, s, parent, token, cum, n):
        BW, S = self.BW, self.S
        paths = np.full_like(self.paths, -1)
        for b in range(n):
            paths[b, :s] = self.paths[parent[b], :s]
            paths[b, s] = token[b]
        self.paths = paths
        self.parents.append(parent.copy())
        self.anc = ancestry_forward(self.anc, parent, s + 1, n)
        self.cum = np.array(cum, dtype=self.cum.dtype)
        self.n_live = n

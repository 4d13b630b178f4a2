"""Test-side driver: run the CUDA path (through the C ABI) and the oracle on the
same seeded inputs, step by step, and compare.

Tolerances (attention): max-abs 2e-2, relative L2 5e-3 over the compared rows,
|dLSE| 1e-3 -- bf16 K/V/Q with fp32 accumulation against fp64.  Masks and the
log-prob selection are compared bit for bit.  Logits-mode selection is
compared tie-aware: a difference is allowed only between candidates whose
fp64 oracle scores are within 1e-4.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

import oracle
import workloads
from shared_prefix_decode_xattention_b200 import xgr
from shared_prefix_decode_xattention_b200.session import Session, config_for

ATOL_O = 2e-2
RL2_O = 5e-3
ATOL_LSE = 1e-3
TIE_EPS = 1e-4


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclasses.dataclass
class StepOut:
    out: torch.Tensor
    lse: torch.Tensor
    mask: tuple
    parent: Optional[np.ndarray] = None
    token: Optional[np.ndarray] = None
    cum: Optional[np.ndarray] = None
    n_out: Optional[np.ndarray] = None


class GpuRun:
    """One decode of workload w on cuda:0 through the C ABI."""

    def __init__(self, w, items=None, device="cuda", max_partials=0, per_beam=False, capacity=None):
        self.w, self.device = w, device
        self.per_beam = per_beam   # attention by the per-beam comparison path
        # capacity: a context sized for more requests than the decode runs
        cw = w if capacity is None else workloads.small(w, B=capacity)
        self.sess = Session(config_for(cw, max_partials=max_partials), device)
        if w.V:
            self.sess.build_trie(items)
        self.kv = {}
        for sid in range(w.n_shared):
            members = [r for r in range(w.B) if w.shared_id(r) == sid]
            if not members:
                continue
            k, v = workloads.shared_kv(w, sid, device)
            self.kv[("s", sid)] = (k, v)
            self.sess.prefill(members[0], sid, k, v)
            for r in members[1:]:
                self.sess.link(r, sid)
        if w.suffix[1]:
            for r in range(w.B):
                k, v = workloads.suffix_kv(w, r, device)
                self.kv[("x", r)] = (k, v)
                self.sess.prefill(r, 0, k, v, kind=xgr.XGR_KV_SUFFIX)
        self.n = w.B      # requests of the current decode
        self.sess.begin(w.B)
        self.kinds = []   # the mask kind of every sparse step

    def restart(self, n: int):
        """A new decode of the context's first n requests (xgr_begin(n))."""
        self.n = n
        self.sess.begin(n)

    def step(self, s, q, kn, vn, scores=None, flags=xgr.XGR_SCORES_LOGPROB) -> StepOut:
        w, B = self.w, self.n
        # NaN sentinels: every row the call must write (dead beams' zeros included) is checked
        out = torch.full((B, w.BW, w.Hq, w.D), float("nan"), dtype=torch.bfloat16, device=self.device)
        lse = torch.full((B, w.BW, w.Hq), float("nan"), dtype=torch.float32, device=self.device)
        if self.per_beam:
            self.sess.decode_step_per_beam(s, q, kn, vn, out, lse)
        else:
            self.sess.decode_step(s, q, kn, vn, out, lse)
        if not w.V:
            return StepOut(out, lse, None)
        m = self.sess.build_mask(s)
        if m.kind == xgr.XGR_MASK_DENSE:
            bits = torch.empty(m.n_words, dtype=torch.int32, device=self.device)
            torch.cuda.synchronize()
            _copy_dev(bits, m.bits, m.n_words * 4, self.sess)
            mask = ("dense", bits.cpu().numpy().view(np.uint32).copy())
        else:
            assert m.kind in (xgr.XGR_MASK_NODE_BITS, xgr.XGR_MASK_TRIE_ROWS), m.kind
            self.kinds.append(m.kind)
            rp, cols = self.sess.mask_csr(m)   # the rows the selection reads, written out
            torch.cuda.synchronize()
            rpn = rp.cpu().numpy()
            nnz = int(rpn[-1])
            mask = ("csr", (rpn.astype(np.int64), cols.cpu().numpy()[:nnz].copy()))
            if m.kind == xgr.XGR_MASK_NODE_BITS:
                _check_node_bits(m, mask[1], w.V, self.sess)
        parent = torch.empty((B, w.BW), dtype=torch.int32, device=self.device)
        token = torch.empty_like(parent)
        cum = torch.empty((B, w.BW), dtype=torch.float32, device=self.device)
        n_out = torch.empty((B,), dtype=torch.int32, device=self.device)
        self.sess.beam_select(s, scores, flags, m, parent, token, cum, n_out)
        torch.cuda.synchronize()
        return StepOut(out, lse, mask, parent.cpu().numpy(), token.cpu().numpy(),
                       cum.cpu().numpy(), n_out.cpu().numpy())

    def sequences(self) -> np.ndarray:
        w = self.w
        seq = torch.empty((self.n, w.BW, w.S), dtype=torch.int32, device=self.device)
        self.sess.sequences(seq)
        torch.cuda.synchronize()
        return seq.cpu().numpy()

    def status(self) -> int:
        return self.sess.device_status()


def _check_node_bits(m, csr, V: int, sess: Session):
    """The pre-generated bitset of every row's node holds exactly that row's
    valid tokens (the CSR rows, themselves compared with the oracle)."""
    nodes = torch.empty(m.n_rows, dtype=torch.int32, device=sess.workspace.device)
    _copy_dev(nodes, m.row_node, m.n_rows * 4, sess)
    off = m.bits - sess.workspace.data_ptr()
    nbytes = m.n_nodes * m.n_words * 4
    assert 0 <= off and off + nbytes <= sess.nbytes
    table = sess.workspace[off:off + nbytes].view(torch.int32).view(m.n_nodes, m.n_words)
    nd = nodes.cpu().numpy()
    rows = np.nonzero(nd >= 0)[0]
    got = table[torch.as_tensor(nd[rows]).long().to(table.device)].cpu().numpy().view(np.uint8)
    dense = np.unpackbits(got, axis=1, bitorder="little")[:, :V].astype(bool)
    rp, cols = csr
    want = np.zeros_like(dense)
    for i, row in enumerate(rows):
        want[i, cols[rp[row]:rp[row + 1]]] = True
    assert np.array_equal(dense, want), "a node's pre-generated bitset differs from its valid tokens"
    for row in np.nonzero(nd < 0)[0]:
        assert rp[row + 1] == rp[row], "a row without a node has tokens"


def _copy_dev(dst: torch.Tensor, src_ptr: int, nbytes: int, sess: Session):
    """Copy a library-owned view (a pointer into the session's workspace tensor)."""
    off = src_ptr - sess.workspace.data_ptr()
    assert 0 <= off and off + nbytes <= sess.nbytes
    dst.view(torch.uint8)[:nbytes].copy_(sess.workspace[off:off + nbytes])


def oracle_request(w, sorted_items, run: GpuRun, r: int, mode="logprob"):
    """Oracle beam decode of request r with the same prompt/suffix KV as the GPU run."""
    ks, vs = run.kv[("s", w.shared_id(r))]
    kx = vx = None
    if ("x", r) in run.kv:
        kx, vx = run.kv[("x", r)]
        kx, vx = u16(kx), u16(vx)
    dec = oracle.BeamDecode(sorted_items, w.BW, w.K, w.S, w.Hq, w.Hkv, w.D, w.V, mode=mode)
    dec.begin(u16(ks), u16(vs), kx, vx)
    return dec


def compare_attention(o_gpu: torch.Tensor, lse_gpu: torch.Tensor, o_ref: np.ndarray,
                      lse_ref: np.ndarray, live: np.ndarray, what=""):
    """o_gpu [n][Hq][D] bf16, lse_gpu [n][Hq]; o_ref, lse_ref fp64; live bool [n]."""
    og = o_gpu.float().cpu().numpy().astype(np.float64)
    lg = lse_gpu.cpu().numpy().astype(np.float64)
    if (~live).any():
        assert np.all(og[~live] == 0), f"{what}: dead rows not zero"
        assert np.all(np.isneginf(lg[~live])), f"{what}: dead LSE not -inf"
    if live.any():
        a, b = og[live], o_ref[live]
        err = np.abs(a - b).max()
        rl2 = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
        lerr = np.abs(lg[live] - lse_ref[live]).max()
        assert err <= ATOL_O, f"{what}: max-abs {err}"
        assert rl2 <= RL2_O, f"{what}: rel-L2 {rl2}"
        assert lerr <= ATOL_LSE, f"{what}: LSE {lerr}"
        return err, rl2, lerr
    return 0.0, 0.0, 0.0


def compare_mask(gpu_mask, ora_mask, r: int, BW: int, what=""):
    kind, data = gpu_mask
    okind, odata = ora_mask
    assert kind == okind, what
    if kind == "dense":
        assert np.array_equal(data, odata), f"{what}: dense mask differs"
        return
    rp, cols = data
    orp, ocols = odata
    for b in range(BW):
        row = r * BW + b
        g = cols[rp[row]:rp[row + 1]]
        o = ocols[orp[b]:orp[b + 1]]
        assert np.array_equal(g, o), f"{what}: mask row {row} differs"


def compare_select_exact(so: StepOut, r: int, parent, token, cum, n, what=""):
    assert so.n_out[r] == n, f"{what}: n_out {so.n_out[r]} vs {n}"
    assert np.array_equal(so.parent[r], parent), f"{what}: parent differs"
    assert np.array_equal(so.token[r], token), f"{what}: token differs"
    assert so.cum[r].tobytes() == np.asarray(cum, np.float32).tobytes(), f"{what}: cum differs"


def compare_select_tie_aware(so: StepOut, r: int, dec, scores_r: np.ndarray, mask, s: int,
                             what=""):
    """Logits mode: the GPU's chosen set may differ from the oracle's only among
    candidates whose fp64 scores are within TIE_EPS; cum within TIE_EPS."""
    row_ptr, cols = dec._rows(s, mask)
    pr, tk, cm, n, _ = oracle.select_logits(dec.cum, scores_r, row_ptr, cols, dec.BW, dec.n_live)
    assert so.n_out[r] == n, what
    gp, gt = so.parent[r][:n], so.token[r][:n]
    # every choice is a distinct candidate of the oracle's mask for this step
    assert len(set(zip(gp.tolist(), gt.tolist()))) == n, f"{what}: a (parent, token) repeats"
    for p_, t_ in zip(gp.tolist(), gt.tolist()):
        assert 0 <= p_ < dec.n_live, f"{what}: parent {p_} not live"
        row = cols[row_ptr[p_]:row_ptr[p_ + 1]] if s else cols
        assert t_ in set(row.tolist()), f"{what}: token {t_} not valid for parent {p_}"
    dead = so.parent[r][n:]
    assert np.all(dead == -1) and np.all(so.token[r][n:] == -1), f"{what}: dead slots"
    gk = oracle.logits_keys(dec.cum, scores_r, list(zip(gp.tolist(), gt.tolist())))
    # -inf is an ordinary (lowest) score: two -inf keys are equal, not NaN apart
    def close(x, y):
        with np.errstate(invalid="ignore"):
            return (x == y) | (np.abs(x - y) <= TIE_EPS)
    # the GPU's k-th choice has the oracle's k-th best score up to near-ties
    assert np.all(close(np.sort(gk)[::-1], cm[:n])), f"{what}: selection differs"
    assert np.all(close(so.cum[r][:n].astype(np.float64), gk)), f"{what}: cum"
    return gp, gt, n

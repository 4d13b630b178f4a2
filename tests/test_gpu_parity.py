"""GPU parity: the CUDA path (through the C ABI) against the oracle, step by
step, on the same seeded inputs, for every workload shape.

Workloads 1, 2 and 4 are compared in full; 3 and 5 on sampled requests (every
selection of the request, a deterministic sample of beams for attention).
Attention within max-abs 2e-2 / rel-L2 5e-3 / LSE 1e-3; masks and log-prob
selections bit-exact; logits-mode selections tie-aware (1e-4).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from harness import (GpuRun, compare_attention, compare_mask, compare_select_exact,
                     compare_select_tie_aware, oracle_request)
from shared_prefix_decode_xattention_b200 import xgr

pytestmark = pytest.mark.gpu


def _sample_beams(n_live, k, seed):
    if k is None or n_live <= k:
        return None
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n_live, size=k, replace=False)).astype(np.int32)


def decode_and_compare(w, mode="logprob", requests=None, beams_per_step=None, items=None,
                       max_partials=0, scores_fn=None, per_beam=False, capacity=None):
    items = workloads.items(w) if items is None else items
    si = oracle.SortedItems(items, w.V) if w.V else None
    run = GpuRun(w, items, max_partials=max_partials, per_beam=per_beam, capacity=capacity)
    reqs = list(range(w.B)) if requests is None else list(requests)
    decs = {r: oracle_request(w, si, run, r, mode) for r in reqs}
    flags = xgr.XGR_SCORES_LOGPROB if mode == "logprob" else xgr.XGR_SCORES_LOGITS
    worst = [0.0, 0.0, 0.0]
    for s in range(w.S):
        q, kn, vn = workloads.step_qkv(w, s, "cuda")
        scores = None
        if w.V:
            if scores_fn is not None:
                scores = scores_fn(s)
            elif mode == "logprob":
                scores = workloads.step_logprobs(w, s, "cuda")
            else:
                scores = workloads.step_logits(w, s, "cuda")
        so = run.step(s, q, kn, vn, scores, flags)
        qc, knc, vnc = q.cpu(), kn.cpu(), vn.cpu()
        sc = scores.cpu().numpy() if scores is not None else None
        for r in reqs:
            dec = decs[r]
            beams = _sample_beams(dec.n_live, beams_per_step, 1000 * s + r)
            o_ref, l_ref = dec.attention(s, qc[r], knc[r], vnc[r], beams)
            ids = np.arange(w.BW) if beams is None else beams
            live = ids < dec.n_live
            errs = compare_attention(so.out[r][torch.as_tensor(ids).long()],
                                     so.lse[r][torch.as_tensor(ids).long()], o_ref, l_ref, live,
                                     f"step {s} request {r}")
            worst = [max(a, b) for a, b in zip(worst, errs)]
            if not w.V:
                continue
            om = dec.mask(s)
            compare_mask(so.mask, om, r, w.BW, f"step {s} request {r}")
            if mode == "logprob":
                p, t, c, n = dec.select(s, sc[r], om)
                compare_select_exact(so, r, p, t, c, n, f"step {s} request {r}")
            else:
                compare_select_tie_aware(so, r, dec, sc[r], om, s, f"step {s} request {r}")
                dec.select(s, sc[r], om, force=(so.parent[r], so.token[r], so.n_out[r]))
    if w.V:
        seq = run.sequences()
        item_set = {tuple(x) for x in items.tolist()}
        for r in reqs:
            dec = decs[r]
            assert np.array_equal(seq[r], dec.paths), f"sequences of request {r}"
            for b in range(dec.n_live):
                assert tuple(seq[r, b].tolist()) in item_set
    assert run.status() == 0
    run.sess.close()
    return worst, run.kinds


def test_workload1_logprob_full():
    decode_and_compare(workloads.WORKLOADS[1])


def test_workload1_logits_tie_aware():
    decode_and_compare(workloads.WORKLOADS[1], mode="logits")


def test_workload2_logprob_full():
    _, kinds = decode_and_compare(workloads.WORKLOADS[2])
    # xGR 2.2 "Hybrid dense/sparse storage": step 1 (about 122 valid tokens per
    # beam out of 8192) takes the pre-generated per-node bitsets, step 2 (about
    # one) the trie rows that the rewiring updates in place
    assert kinds == [xgr.XGR_MASK_NODE_BITS, xgr.XGR_MASK_TRIE_ROWS]


def test_workload2_logits_sampled():
    decode_and_compare(workloads.WORKLOADS[2], mode="logits", requests=[0, 5],
                       beams_per_step=16)


def test_workload3_sampled():
    decode_and_compare(workloads.WORKLOADS[3], requests=[0, 13, 22, 31], beams_per_step=12)


def test_workload3_logits_sampled():
    """Logits mode at the 512x512 pool: row log-sum-exp over V = 8192, about 475
    valid tokens per beam at step 1 (beams whose whole head survives the
    threshold, so their further keys are read)."""
    decode_and_compare(workloads.WORKLOADS[3], mode="logits", requests=[3, 30], beams_per_step=8)


def test_workload5_logits_sampled():
    """Logits mode over V = 16384 with ragged long prompts and four steps."""
    decode_and_compare(workloads.WORKLOADS[5], mode="logits", requests=[7, 100],
                       beams_per_step=6)


def test_workload4_homogeneous():
    decode_and_compare(workloads.WORKLOADS[4])


def test_workload4_heterogeneous_sampled():
    w = workloads.heterogeneous(workloads.WORKLOADS[4])
    decode_and_compare(w, requests=[0, 9, 17, 30, 41, 50, 58, 63])


def test_workload5_sampled():
    decode_and_compare(workloads.WORKLOADS[5], requests=[0, 41, 90, 127], beams_per_step=8)


# ------------------------------------------------------------------ edges

def test_ragged_prompts_and_split_k():
    """Prompt lengths that are not multiples of any tile (1 .. 700 tokens), and
    several requests per shared prefix so split-K partials are merged."""
    w = workloads.small(workloads.WORKLOADS[1], wid=101, B=6, prompt=(1, 700), BW=8, K=9,
                        Hq=8, Hkv=2, D=128)
    decode_and_compare(w)
    w2 = workloads.small(workloads.WORKLOADS[4], wid=102, B=8, groups=2, prompt=(1000, 1000),
                         suffix=(1, 300), Hq=16, Hkv=4)
    decode_and_compare(w2, max_partials=6)


def test_unshared_staging_in_batches():
    """The tensor-core kernel gathers each tile's beams' own k/v rows into
    128-row Unshared chunks; when the tile's beams x tokens pass 128 it runs
    several chunks through the same U area.  G = 1 (128 beams in a 128-row
    tile: up to three chunks at step 2) and G = 2 over six steps (64 beams, up
    to three chunks)."""
    w = workloads.small(workloads.WORKLOADS[1], wid=105, B=2, prompt=(300, 300), BW=128, K=128,
                        S=3, Hq=4, Hkv=4, D=128, V=256, n_items=20000)
    decode_and_compare(w, beams_per_step=16)
    w2 = workloads.small(workloads.WORKLOADS[1], wid=106, B=2, prompt=(200, 200), BW=64, K=64,
                         S=6, Hq=4, Hkv=2, D=128, V=64, n_items=30000)
    decode_and_compare(w2, beams_per_step=16)


def test_shared_prefix_groups_with_beams():
    """Beam search over requests that share prompts in groups: one KV segment
    with several member requests per 128-row tile (Q staged by the threads, not
    one TMA box; the staged Unshared rows of two requests in one tile) and, at
    step 0, the zero fill of every member's beams that are not live yet."""
    w = workloads.small(workloads.WORKLOADS[2], wid=107, B=4, groups=2, prompt=(600, 600), BW=16,
                        K=16, S=3, Hq=8, Hkv=2, D=128, V=512, n_items=20000)
    decode_and_compare(w)


def test_largest_beam_width_and_vocabulary():
    """The configuration's limits: BW = K = 1024 (each beam's ordered head
    shrinks to 4 keys; the pick's survivor buffer is at its largest) over a
    32768-token vocabulary (the largest the selection takes: its dense first
    step stages the whole row), in both score modes; attention on a sample of
    beams."""
    w = workloads.small(workloads.WORKLOADS[1], wid=108, B=2, prompt=(256, 256), BW=1024, K=1024,
                        S=3, Hq=4, Hkv=1, D=128, V=32768, n_items=200000)
    decode_and_compare(w, beams_per_step=16)
    decode_and_compare(w, mode="logits", beams_per_step=16)


def test_longest_items():
    """Eight-token items, the most decode steps a context takes: at the last
    step every beam attends to eight Unshared tokens through its ancestry (16
    beams x 8 tokens fill one 128-row Unshared chunk at G = 2), in both score
    modes."""
    w = workloads.small(workloads.WORKLOADS[1], wid=109, B=2, prompt=(300, 300), BW=16, K=16,
                        S=8, Hq=4, Hkv=2, D=128, V=64, n_items=5000)
    decode_and_compare(w)
    decode_and_compare(w, mode="logits")


def test_fewer_requests_than_the_context_holds():
    """A context sized for 8 requests decoding a batch of 3: the beam state and
    the Unshared pool keep the capacity's strides while the work plan, the
    masks and the selection cover the 3 requests of this decode."""
    w = workloads.small(workloads.WORKLOADS[2], wid=110, B=3, prompt=(500, 500), n_items=200000)
    decode_and_compare(w, capacity=8, beams_per_step=16)
    decode_and_compare(w, mode="logits", capacity=8, beams_per_step=16)


def test_context_reused_across_batch_sizes():
    """One context decodes its first 3 requests, then all 8, then 3 again:
    every xgr_begin re-plans for its batch and resets the beam state, so each
    decode matches the oracle (log-prob mode, selections and final sequences
    bit-exact) whatever the decodes before it left in the workspace."""
    w = workloads.small(workloads.WORKLOADS[2], wid=112, B=8, prompt=(400, 400), n_items=200000)
    items = workloads.items(w)
    si = oracle.SortedItems(items, w.V)
    run = GpuRun(w, items)
    inputs = [(*workloads.step_qkv(w, s, "cuda"), workloads.step_logprobs(w, s, "cuda"))
              for s in range(w.S)]
    for n in (3, 8, 3):
        run.restart(n)
        decs = {r: oracle_request(w, si, run, r) for r in sorted({0, n - 1})}
        for s in range(w.S):
            q, kn, vn, lp = (t[:n].contiguous() for t in inputs[s])
            so = run.step(s, q, kn, vn, lp)
            qc, knc, vnc, sc = q.cpu(), kn.cpu(), vn.cpu(), lp.cpu().numpy()
            for r, dec in decs.items():
                what = f"batch of {n}, step {s}, request {r}"
                beams = _sample_beams(dec.n_live, 8, 1000 * s + r)
                o_ref, l_ref = dec.attention(s, qc[r], knc[r], vnc[r], beams)
                ids = np.arange(w.BW) if beams is None else beams
                idx = torch.as_tensor(ids).long()
                compare_attention(so.out[r][idx], so.lse[r][idx], o_ref, l_ref, ids < dec.n_live, what)
                om = dec.mask(s)
                compare_mask(so.mask, om, r, w.BW, what)
                p, t, c, cnt = dec.select(s, sc[r], om)
                compare_select_exact(so, r, p, t, c, cnt, what)
        seq = run.sequences()
        for r, dec in decs.items():
            assert np.array_equal(seq[r], dec.paths), f"batch of {n}: sequences of request {r}"
    assert run.status() == 0
    run.sess.close()


def test_logits_of_large_magnitude_and_minus_inf():
    """Logits mode on rows whose unshifted exponentials overflow fp32: logits of
    spread 20 around 100 (kept below a few hundred so that one fp32 ulp of the
    row's log-sum-exp stays under the 1e-4 tie tolerance), and every seventh
    token at -inf (a score that ranks last; it adds nothing to a row's
    log-sum-exp).  The tiny workload in full, and two requests of the 128-beam
    pool (its streamed rows and dense first step)."""
    def extreme(w):
        def fn(s):
            x = workloads.step_logits(w, s, "cuda") * 10.0 + 100.0
            x[..., ::7] = float("-inf")
            return x
        return fn
    w1 = workloads.WORKLOADS[1]
    decode_and_compare(w1, mode="logits", scores_fn=extreme(w1))
    w2 = workloads.WORKLOADS[2]
    decode_and_compare(w2, mode="logits", requests=[1, 6], beams_per_step=8, scores_fn=extreme(w2))


def test_logprob_minus_inf_scores():
    """Log-prob mode with every fifth token at -inf (a token the model rules
    out): such candidates rank after every finite one and among themselves by
    parent, then token; selections bit-exact.  Two requests of the 128-beam
    pool, where late steps have about one valid token per beam, so -inf
    candidates are among the winners."""
    w = workloads.WORKLOADS[2]

    def fn(s):
        x = workloads.step_logprobs(w, s, "cuda")
        x[..., ::5] = float("-inf")
        return x
    decode_and_compare(w, requests=[2, 7], beams_per_step=8, scores_fn=fn)


def test_fewer_candidates_than_beams():
    """A vocabulary of 3 items: at most 3 live beams of 8, the rest dead."""
    w = workloads.small(workloads.WORKLOADS[1], wid=103, BW=8, K=8, n_items=3)
    decode_and_compare(w)


def test_all_scores_tied_fallback_path():
    """Every score equal: the ordering falls to parent then token, and the
    survivors of the threshold exceed the sort buffer (exact radix fallback)."""
    w = workloads.small(workloads.WORKLOADS[2], wid=104, B=2)
    tie = lambda s: torch.full((w.B, w.BW, w.V), -9.0, device="cuda")
    decode_and_compare(w, scores_fn=tie, beams_per_step=4)


def test_nan_score_sets_device_status():
    w = workloads.WORKLOADS[1]
    items = workloads.items(w)
    run = GpuRun(w, items)
    q, kn, vn = workloads.step_qkv(w, 0, "cuda")
    lp = workloads.step_logprobs(w, 0, "cuda")
    lp[0, 0, int(items[0, 0])] = float("nan")
    run.step(0, q, kn, vn, lp)
    assert run.status() & xgr.XGR_DEV_NAN
    assert run.status() == 0   # cleared by the read


def test_abi_call_order_and_arguments():
    w = workloads.WORKLOADS[1]
    items = workloads.items(w)
    run = GpuRun(w, items)
    q, kn, vn = workloads.step_qkv(w, 0, "cuda")
    out = torch.empty((w.B, w.BW, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.BW, w.Hq), dtype=torch.float32, device="cuda")
    with pytest.raises(xgr.XgrError) as e:
        run.sess.decode_step(1, q, kn, vn, out, lse)           # step 1 before step 0
    assert e.value.status == xgr.XGR_ERR_STATE
    with pytest.raises(xgr.XgrError) as e:
        run.sess.decode_step(0, q.data_ptr() + 2, kn, vn, out, lse)   # misaligned
    assert e.value.status == xgr.XGR_ERR_ARG
    with pytest.raises(xgr.XgrError) as e:
        xgr.xgr_build_trie(run.sess.ctx, items[:, :2])         # wrong item length
    assert e.value.status == xgr.XGR_ERR_SHAPE
    big = torch.zeros((w.Hkv, 10_000, w.D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(xgr.XgrError) as e:
        run.sess.prefill(0, 0, big, big)                      # store too small
    assert e.value.status == xgr.XGR_ERR_CAPACITY
    m = run.sess.build_mask(0)
    p = torch.empty((w.B, w.BW), dtype=torch.int32, device="cuda")
    c = torch.empty((w.B, w.BW), dtype=torch.float32, device="cuda")
    n = torch.empty((w.B,), dtype=torch.int32, device="cuda")
    lp = workloads.step_logprobs(w, 0, "cuda")
    with pytest.raises(xgr.XgrError) as e:
        run.sess.beam_select(0, lp, 7, m, p, p.clone(), c, n)   # unknown flag
    assert e.value.status == xgr.XGR_ERR_ARG
    assert run.status() == 0

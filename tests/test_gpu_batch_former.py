"""GPU: batches formed by the Chunked Hash Tree feed the staged attention.

Feather page ("Requests of the same feather must flock together"),
"Methodology", 1. Chunked Hash Tree, and "Results": prefix-homogeneous batches
are the ones whose shared prefix is read once for all members.  Here the 64
requests of the prefix-shared workload (4 prompt families of 16, 8192-token
family prefixes, private suffixes of 256-2048 tokens) arrive in a shuffled
order; the tree forms the batches; each batch becomes one shared KV segment
(its first member's prefix, as deep as the batch shares it) that every member
links to, with the rest of each prompt loaded as the member's private suffix;
one decode step runs through the C ABI and every request's attention is
compared with the oracle over that request's own full prompt.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from harness import compare_attention, u16
from shared_prefix_decode_xattention_b200 import xgr
from shared_prefix_decode_xattention_b200.sched import ChunkedHashTree
from shared_prefix_decode_xattention_b200.session import Session, config_for

pytestmark = pytest.mark.gpu

CHUNK = 256


def _prompt_tokens(w):
    """Token ids of every request's prompt: its family's prefix, then its own suffix."""
    rng = np.random.default_rng(4242)
    lens = workloads.prompt_lengths(w)
    fam = [rng.integers(0, 32000, size=int(lens[g])) for g in range(w.n_shared)]
    suf = workloads.suffix_lengths(w)
    return [np.concatenate([fam[w.shared_id(r)], rng.integers(0, 32000, size=int(suf[r]))])
            for r in range(w.B)]


def test_tree_batches_feed_the_attention():
    w = workloads.WORKLOADS[4]
    toks = _prompt_tokens(w)
    tree = ChunkedHashTree(CHUNK)
    for r in np.random.default_rng(7).permutation(w.B):   # interleaved arrivals
        tree.insert(int(r), toks[r])
    batches = tree.form_batches(w.B // w.groups, 1)
    # the four families come back whole, each sharing its full prefix
    assert sorted(sorted(m) for m, _ in batches) == [
        list(range(g * 16, g * 16 + 16)) for g in range(w.groups)]
    assert all(sh * CHUNK == int(workloads.prompt_lengths(w)[0]) for _, sh in batches)

    # the families' prefix K/V and the requests' suffix K/V (drawn once on the
    # device; the oracle reads the same tensors)
    fam_kv = {g: workloads.shared_kv(w, g, "cuda") for g in range(w.groups)}
    suf_kv = {r: workloads.suffix_kv(w, r, "cuda") for r in range(w.B)}
    sess = Session(config_for(w), "cuda")
    for sid, (members, shared_chunks) in enumerate(batches):
        depth = shared_chunks * CHUNK
        k, v = fam_kv[w.shared_id(members[0])]   # the batch's prefix: its first member's
        sess.prefill(members[0], sid, k[:, :depth].contiguous(), v[:, :depth].contiguous())
        for r in members[1:]:
            sess.link(r, sid)
    for r in range(w.B):
        sess.prefill(r, 0, *suf_kv[r], kind=xgr.XGR_KV_SUFFIX)
    sess.begin(w.B)
    q, kn, vn = workloads.step_qkv(w, 0, "cuda")
    out = torch.full((w.B, w.BW, w.Hq, w.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.B, w.BW, w.Hq), float("nan"), dtype=torch.float32, device="cuda")
    sess.decode_step(0, q, kn, vn, out, lse)
    torch.cuda.synchronize()
    qc, knc, vnc = q.cpu(), kn.cpu(), vn.cpu()
    for r in range(w.B):
        ks, vs = fam_kv[w.shared_id(r)]   # the request's own full prompt
        kx, vx = suf_kv[r]
        dec = oracle.BeamDecode(None, w.BW, w.K, w.S, w.Hq, w.Hkv, w.D, w.V)
        dec.begin(u16(ks), u16(vs), u16(kx), u16(vx))
        o_ref, l_ref = dec.attention(0, qc[r], knc[r], vnc[r])
        compare_attention(out[r], lse[r], o_ref, l_ref, np.ones(w.BW, bool), f"request {r}")
    assert sess.device_status() == 0
    sess.close()


@pytest.mark.parametrize("batching", ["tree", "arrival_order"])
def test_batches_as_separate_contexts(batching):
    """The launch configurations the bench times: each batch of 16 requests is
    a context of its own.  A tree batch holds one shared 8192-token prefix
    beside 16 private suffixes, so the work plan splits the prefix into
    several key ranges (it is more than twice the average key load per SM)
    and the merge kernel folds them with each suffix; a batch of consecutive
    arrivals holds the four families' prefixes, each linked by its own
    members.  Every request's attention is compared with the oracle over its
    own full prompt."""
    w = workloads.WORKLOADS[4]
    toks = _prompt_tokens(w)
    arrivals = [int(r) for r in np.random.default_rng(7).permutation(w.B)]
    lens, suf = workloads.prompt_lengths(w), workloads.suffix_lengths(w)
    if batching == "tree":
        tree = ChunkedHashTree(CHUNK)
        for r in arrivals:
            tree.insert(r, toks[r])
        formed = tree.form_batches(w.B // w.groups, 1)
        tree.close()
        for members, shared_chunks in formed:
            assert shared_chunks * CHUNK == int(lens[w.shared_id(members[0])])
        batches = [list(m) for m, _ in formed]
    else:
        batches = [arrivals[i:i + 16] for i in range(0, w.B, 16)]
    q, kn, vn = workloads.step_qkv(w, 0, "cuda")
    qc, knc, vnc = q.cpu(), kn.cpu(), vn.cpu()
    fam_kv = {g: workloads.shared_kv(w, g, "cuda") for g in range(w.groups)}
    for members in batches:
        n = len(members)
        fams = sorted({w.shared_id(r) for r in members})
        cfg = xgr.make_config(max_requests=n, max_shared=len(fams),
                              kv_tokens=sum(int(lens[g]) for g in fams) + sum(int(suf[r]) for r in members),
                              beam_width=1, top_k=1, steps=1, n_q_heads=w.Hq, n_kv_heads=w.Hkv,
                              head_dim=w.D, vocab=0, max_items=0, max_fanout=0, max_partials=0)
        sess = Session(cfg, "cuda")
        for sid, g in enumerate(fams):
            idx = [i for i, r in enumerate(members) if w.shared_id(r) == g]
            sess.prefill(idx[0], sid, *fam_kv[g])
            for i in idx[1:]:
                sess.link(i, sid)
        suf_kv = {r: workloads.suffix_kv(w, r, "cuda") for r in members}
        for i, r in enumerate(members):
            sess.prefill(i, 0, *suf_kv[r], kind=xgr.XGR_KV_SUFFIX)
        sel = torch.tensor(members, device="cuda")
        out = torch.full((n, 1, w.Hq, w.D), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((n, 1, w.Hq), float("nan"), dtype=torch.float32, device="cuda")
        sess.begin(n)
        sess.decode_step(0, q[sel].contiguous(), kn[sel].contiguous(), vn[sel].contiguous(), out, lse)
        torch.cuda.synchronize()
        assert sess.device_status() == 0
        for i, r in enumerate(members):
            ks, vs = fam_kv[w.shared_id(r)]
            kx, vx = suf_kv[r]
            dec = oracle.BeamDecode(None, w.BW, w.K, w.S, w.Hq, w.Hkv, w.D, w.V)
            dec.begin(u16(ks), u16(vs), u16(kx), u16(vx))
            o_ref, l_ref = dec.attention(0, qc[r], knc[r], vnc[r])
            compare_attention(out[i], lse[i], o_ref, l_ref, np.ones(w.BW, bool), f"request {r}")
        sess.close()

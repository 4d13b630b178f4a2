"""The whole-decode graph (xgr_decode_graph_*, include/xgr.h): a decode of
several request groups, each with its own context and stream, captured once
and launched as one graph.  Its results must be those of the same decode
issued call by call -- bit for bit, the kernels being the same -- on every
launch, for one, two and four groups of the 128-beam workload (whose eager
decode the parity tests compare with the oracle), in both score modes."""
import pytest
import torch

import workloads
from shared_prefix_decode_xattention_b200 import xgr
from shared_prefix_decode_xattention_b200.session import Session, config_for


def _groups(w, G, dev, flags):
    Bg = w.B // G
    wg = workloads.small(w, B=Bg)
    items = workloads.items(w)
    gen = workloads.step_logits if flags == xgr.XGR_SCORES_LOGITS else workloads.step_logprobs
    inputs = [workloads.step_qkv(w, s, dev) + (gen(w, s, dev),) for s in range(w.S)]
    groups = []
    for g in range(G):
        sess = Session(config_for(wg), dev)
        sess.build_trie(items)
        for i in range(Bg):
            k, v = workloads.shared_kv(w, w.shared_id(g * Bg + i), dev)
            sess.prefill(i, i, k, v)
        sl = slice(g * Bg, (g + 1) * Bg)
        groups.append(dict(
            sess=sess, ctx=sess.ctx, n_requests=Bg, score_flags=flags,
            q=[x[0][sl] for x in inputs], k_new=[x[1][sl] for x in inputs],
            v_new=[x[2][sl] for x in inputs], scores=[x[3][sl] for x in inputs],
            out=torch.empty((Bg, w.BW, w.Hq, w.D), dtype=torch.bfloat16, device=dev),
            lse=torch.empty((Bg, w.BW, w.Hq), dtype=torch.float32, device=dev),
            parent=torch.empty((Bg, w.BW), dtype=torch.int32, device=dev),
            token=torch.empty((Bg, w.BW), dtype=torch.int32, device=dev),
            cum=torch.empty((Bg, w.BW), dtype=torch.float32, device=dev),
            n_out=torch.empty((Bg,), dtype=torch.int32, device=dev)))
    return groups


def _results(w, g):
    seq = torch.empty((g["n_requests"], w.BW, w.S), dtype=torch.int32, device="cuda")
    g["sess"].sequences(seq)
    torch.cuda.synchronize()
    return [t.clone() for t in (g["out"], g["lse"], g["parent"], g["token"], g["cum"], g["n_out"], seq)]


def _eager(w, g):
    s_ = g["sess"]
    s_.begin(g["n_requests"])
    for s in range(w.S):
        m = s_.build_mask(s)
        s_.decode_step(s, g["q"][s], g["k_new"][s], g["v_new"][s], g["out"], g["lse"])
        s_.beam_select(s, g["scores"][s], g["score_flags"], m, g["parent"], g["token"], g["cum"], g["n_out"])
    return _results(w, g)


def _same(a, b):
    for x, y in zip(a, b):
        assert x.shape == y.shape
        assert torch.equal(x.view(torch.uint8) if x.dtype != torch.bfloat16 else x.view(torch.int16),
                           y.view(torch.uint8) if y.dtype != torch.bfloat16 else y.view(torch.int16))


@pytest.mark.gpu
@pytest.mark.parametrize("G,flags", [(1, xgr.XGR_SCORES_LOGITS), (2, xgr.XGR_SCORES_LOGITS),
                                     (4, xgr.XGR_SCORES_LOGPROB)])
def test_decode_graph_equals_the_eager_decode(G, flags):
    w = workloads.WORKLOADS[2]
    groups = _groups(w, G, "cuda", flags)
    want = [_eager(w, g) for g in groups]
    graph = xgr.xgr_decode_graph_create(groups, w.S)
    try:
        # one decode per group: begin, then S x (attention launches + selection launches)
        assert xgr.xgr_decode_graph_kernels(graph) >= G * (1 + 2 * w.S)
        for launch in range(2):
            for g in groups:   # poison the outputs: the launch must rewrite them
                for k in ("out", "lse", "parent", "token", "cum", "n_out"):
                    g[k].fill_(-7 if g[k].dtype != torch.bfloat16 else 0)
            st = torch.cuda.Stream()
            xgr.xgr_decode_graph_launch(graph, st)
            st.synchronize()
            for g, ref in zip(groups, want):
                _same(_results(w, g), ref)
                assert g["sess"].device_status() == 0
    finally:
        xgr.xgr_decode_graph_destroy(graph)
        for g in groups:
            g["sess"].close()

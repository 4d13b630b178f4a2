"""xgr_beam_topk_noalloc: the masked top-K for callers that cannot allocate.

Some callers may not call cudaMalloc or hand the library a workspace (a host
framework that owns every device byte, a plugin that must not allocate after
start-up).  For them the library offers a context-free selection whose
scratch is a fixed static device array.  These tests check that it returns
exactly what the context entry point xgr_beam_select returns -- bit for bit,
the tolerance every selection test here uses -- on two selections in a row
(first step with the dense mask, second step with the CSR masks), in log-prob
and in logits mode, and that its limits are enforced on the host.
"""
import ctypes

import pytest
import torch

import workloads
from shared_prefix_decode_xattention_b200 import build, xgr


def test_noalloc_rejects_bad_arguments_on_the_host():
    build.build()
    L = xgr.lib()
    fake = 1 << 20   # never dereferenced: validation happens before any device work
    args = lambda B, BW, K, V: (B, BW, K, V, fake, 0, fake, fake, fake, None, None,
                                fake, fake, fake, fake, None)
    # 128 requests over V = 16384 need about 25 MiB of scratch: beyond the fixed 8 MiB
    assert L.xgr_beam_topk_noalloc(*args(128, 256, 256, 16384)) == xgr.XGR_ERR_CAPACITY
    assert L.xgr_beam_topk_noalloc(*args(8, 128, 64, 8192)) == xgr.XGR_ERR_SHAPE   # K < BW
    bad = list(args(8, 128, 128, 8192))
    bad[4] = None
    assert L.xgr_beam_topk_noalloc(*bad) == xgr.XGR_ERR_ARG
    bad = list(args(8, 128, 128, 8192))
    bad[5] = 3
    assert L.xgr_beam_topk_noalloc(*bad) == xgr.XGR_ERR_ARG


# the configuration's limits: 1024 beams over a 32768-token vocabulary (each
# beam's head holds 4 keys; the dense step stages the whole row)
_LIMITS = dict(wid=108, B=2, prompt=(256, 256), BW=1024, K=1024, S=3, Hq=4, Hkv=1, D=128,
               V=32768, n_items=200000)


@pytest.mark.gpu
@pytest.mark.parametrize("wid,flags", [(1, xgr.XGR_SCORES_LOGPROB), (2, xgr.XGR_SCORES_LOGITS),
                                       ("limits", xgr.XGR_SCORES_LOGPROB)])
def test_noalloc_matches_context_select(wid, flags):
    from harness import GpuRun
    w = (workloads.small(workloads.WORKLOADS[1], **_LIMITS) if wid == "limits"
         else workloads.WORKLOADS[wid])
    run = GpuRun(w, workloads.items(w))
    B, BW = w.B, w.BW
    dev = "cuda"
    cum = torch.full((B, BW), float("-inf"), device=dev)
    cum[:, 0] = 0.0
    n_live = torch.ones((B,), dtype=torch.int32, device=dev)
    out = torch.empty((B, BW, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, BW, w.Hq), dtype=torch.float32, device=dev)
    for s in range(2):
        q, kn, vn = workloads.step_qkv(w, s, dev)
        gen = workloads.step_logprobs if flags == xgr.XGR_SCORES_LOGPROB else workloads.step_logits
        scores = gen(w, s, dev)
        run.sess.decode_step(s, q, kn, vn, out, lse)
        m = run.sess.build_mask(s)
        want = [torch.empty((B, BW), dtype=torch.int32, device=dev),
                torch.empty((B, BW), dtype=torch.int32, device=dev),
                torch.empty((B, BW), dtype=torch.float32, device=dev),
                torch.empty((B,), dtype=torch.int32, device=dev)]
        got = [torch.full_like(t, 7) for t in want]
        dense = m.kind == xgr.XGR_MASK_DENSE
        rp = cols = None
        if not dense:   # the same rows as explicit CSR, the form this call takes
            rp, cols = run.sess.mask_csr(m)
        run.sess.beam_select(s, scores, flags, m, *want)
        xgr.xgr_beam_topk_noalloc(B, BW, w.K, w.V, scores, flags, cum, n_live,
                                  m.bits if dense else None, rp, cols, *got)
        torch.cuda.synchronize()
        for a, b in zip(want, got):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32)), f"step {s}"
        assert int(want[3].min()) > 0
        cum, n_live = want[2].clone(), want[3].clone()
    assert run.status() == 0
    run.sess.close()

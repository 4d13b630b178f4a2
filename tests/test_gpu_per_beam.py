"""GPU: the per-beam comparison path (xgr_decode_step_per_beam) against the oracle.

xGR page, 1 "Problem definition" (serving systems treat each beam as an
independent sequence: the shared prompt KV is reloaded per beam and blocks are
copied when beams fork) and 4 "Kernel efficiency" (the staged kernel against
that baseline).  The baseline must compute the same attention as the staged
path -- the oracle's unsplit softmax over prompt + suffix + the beam's own
tokens -- with the same tolerances, through whole decodes in which beams fork
(each new beam's block is its parent's, copied, plus this step's token).
"""
import pytest
import torch

import workloads
from shared_prefix_decode_xattention_b200 import xgr
from shared_prefix_decode_xattention_b200.session import Session, config_for
from test_gpu_parity import decode_and_compare

pytestmark = pytest.mark.gpu


def test_per_beam_workload2_decode():
    """128 beams per request fork at every step (sampled requests and beams)."""
    decode_and_compare(workloads.WORKLOADS[2], requests=[0, 3, 7], beams_per_step=24, per_beam=True)


def test_per_beam_prefix_groups_with_suffixes():
    """Workload 4: prompts shared in groups plus private suffixes, beam 1."""
    decode_and_compare(workloads.WORKLOADS[4], requests=[0, 17, 40, 63], per_beam=True)


def test_per_beam_ragged_and_dead_beams():
    """Ragged prompts (1 .. 700 tokens), G = 2, and fewer candidates than beams
    (dead beams: O = 0, LSE = -inf)."""
    w = workloads.small(workloads.WORKLOADS[1], wid=111, B=5, prompt=(1, 700), BW=8, K=8,
                        Hq=8, Hkv=4, D=128, V=256, n_items=6)
    decode_and_compare(w, per_beam=True)


def test_per_beam_argument_checks():
    w = workloads.WORKLOADS[2]
    sess = Session(config_for(w), "cuda")
    k, v = workloads.shared_kv(w, 0, "cuda")
    sess.prefill(0, 0, k, v)
    sess.begin(1)
    q, kn, vn = workloads.step_qkv(w, 0, "cuda")
    out = torch.empty((w.B, w.BW, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.BW, w.Hq), dtype=torch.float32, device="cuda")
    n = xgr.xgr_per_beam_bytes(sess.ctx)
    small = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    with pytest.raises(xgr.XgrError) as e:
        xgr.xgr_decode_step_per_beam(sess.ctx, 0, q, kn, vn, out, lse, small, small.numel())
    assert e.value.status == xgr.XGR_ERR_CAPACITY
    with pytest.raises(xgr.XgrError) as e:
        sess.decode_step_per_beam(1, q, kn, vn, out, lse)   # step 1 before step 0
    assert e.value.status == xgr.XGR_ERR_STATE
    assert sess.device_status() == 0
    sess.close()

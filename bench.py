#!/usr/bin/env python
"""Benchmark of the beam-decode hot path; prints ONE JSON line.

A step is one whole beam decode of a batch: xgr_begin, then for every decode
step s: staged attention (xgr_decode_step), the valid-path mask
(xgr_build_mask) and the masked top-K with rewiring (xgr_beam_select).  The
default workload is the 128x128 candidate pool (8 requests, 1024-token
prompts, beam width = top-K = 128, 3 steps, Hq=16, Hkv=4, D=128, V=8192, 1M
valid 3-token items), logits-mode scores.

metric: beam-candidates/s = sum over decode steps of (requests x live beams x K)
        per second of device time (L2 flushed before every timed step).
--impl reference: the CPU oracle timed on the host cores, same metric.
Multi-GPU (torchrun): every rank decodes its own batch (weak scaling, no
collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "beam-candidates/s per decode step"
UNIT = "candidates/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="xgr", choices=["xgr", "reference"])
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--scores", default="logits", choices=["logits", "logprob"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bw512", action="store_true",
                    help="skip the BW = 512 attention figure (second half of the metric)")
    ap.add_argument("--groups", type=int, default=1,
                    help="request groups decoded on their own streams inside the one graph")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the prefix-batch and long-history workload figures")
    return ap.parse_args()


def workload_config(w, scores):
    return {
        "workload": f"{w.name}: B={w.B} requests, prompt {w.prompt[0]}-{w.prompt[1]} tokens, "
                    f"BW={w.BW}, top-K={w.K}, {w.S} steps, Hq={w.Hq}, Hkv={w.Hkv}, D={w.D}, "
                    f"V={w.V}, {w.n_items} valid items",
        "scores": scores,
        "l2": "flushed (256 MiB write) before every timed step; step time from CUDA events",
        "execution": "each decode replayed as one CUDA graph (per-phase graphs for the breakdown)",
    }


def candidates_per_decode(w):
    return sum(w.candidates_per_step(s) for s in range(w.S))


# ---------------------------------------------------------------- clocks

class Clocks:
    """SM clock and clock-event reasons sampled while the timed region runs:
    NVML polled from a background thread every half millisecond (the timed
    region can be a few milliseconds), else nvidia-smi every 200 ms.  Only
    reads the GPU's state."""
    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("sw_power_cap", 0x4))
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        import threading
        self.sm, self.mx, self.reasons = [], 0.0, set()
        self.p = self.t = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            pr = torch.cuda.get_device_properties(index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.mx = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            self.stop_ev = threading.Event()

            def poll():
                while not self.stop_ev.is_set():
                    try:
                        self.sm.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                        bits = get_reasons(h) if get_reasons else 0
                        for n, b in self.REASONS:
                            if bits & b:
                                self.reasons.add(n)
                    except Exception:
                        return
                    self.stop_ev.wait(0.0005)

            self.t = threading.Thread(target=poll, daemon=True)
            self.t.start()
            return
        except Exception:
            self.t = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.t is not None:
            self.stop_ev.set()
            self.t.join(timeout=5)
            sm = self.sm
        elif self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except Exception:
                self.p.kill()
            self.f.flush()
            rows = [l.strip().split(", ") for l in open(self.f.name) if l.strip()]
            os.unlink(self.f.name)
            sm = []
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for r in rows:
                try:
                    sm.append(float(r[0]))
                    self.mx = max(self.mx, float(r[1]))
                    for n, v in zip(names, r[3:7]):
                        if v.strip().lower() == "active":
                            self.reasons.add(n)
                except (ValueError, IndexError):
                    continue
        else:
            return None
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.mx,
                "reasons": sorted(self.reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle

def oracle_decode_sample(w, items, sorted_items, requests, scores_mode):
    """One full oracle decode of the given requests; returns (seconds, candidates)."""
    import numpy as np
    import torch
    import oracle
    import workloads
    u16 = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    mode = "logprob" if scores_mode == "logprob" else "logits"
    inputs = []
    for s in range(w.S):
        q, kn, vn = workloads.step_qkv(w, s, "cpu")
        sc = (workloads.step_logprobs if mode == "logprob" else workloads.step_logits)(w, s, "cpu")
        inputs.append((q, kn, vn, sc.numpy()))
    kvs = {r: workloads.shared_kv(w, w.shared_id(r), "cpu") for r in requests}
    t0 = time.perf_counter()
    cands = 0
    for r in requests:
        dec = oracle.BeamDecode(sorted_items, w.BW, w.K, w.S, w.Hq, w.Hkv, w.D, w.V, mode=mode)
        k, v = kvs[r]
        dec.begin(u16(k), u16(v))
        for s in range(w.S):
            q, kn, vn, sc = inputs[s]
            cands += dec.n_live * w.K
            dec.attention(s, q[r], kn[r], vn[r])
            m = dec.mask(s)
            dec.select(s, sc[r], m)
    return time.perf_counter() - t0, cands


def cpu_baseline(w, items, scores_mode, budget_s=20.0):
    """The oracle on the host cores: whole decodes of requests 0, 1, ... (then
    of the whole batch again) until about budget_s/2 of all-core time, then
    request 0 with one thread."""
    import oracle
    si = oracle.SortedItems(items, w.V)
    cores = oracle.num_threads()
    secs, cands = oracle_decode_sample(w, items, si, [0], scores_mode)
    reqs = [0]
    r = 1
    while secs < budget_s / 2 and r < w.B:          # grow the sample while it stays short
        t, c = oracle_decode_sample(w, items, si, [r], scores_mode)
        secs += t
        cands += c
        reqs.append(r)
        r += 1
    rounds = 1
    while secs < budget_s / 2:                      # the whole batch fits: repeat it
        t, c = oracle_decode_sample(w, items, si, reqs, scores_mode)
        secs += t
        cands += c
        rounds += 1
    single = None
    try:
        oracle.set_num_threads(1)
        t1, c1 = oracle_decode_sample(w, items, si, reqs[:1], scores_mode)
        single = {"value": c1 / t1, "cores": 1,
                  "sample": f"full {w.S}-step decode of request 0 ({c1} candidates in {t1:.2f} s)"}
    finally:
        oracle.set_num_threads(cores)
    return {"value": cands / secs, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"full {w.S}-step decode of {len(reqs)} of {w.B} requests"
                      + (f", {rounds} times" if rounds > 1 else "")
                      + f" ({cands} candidates in {secs:.2f} s)",
            "single_thread": single}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    import workloads
    items = workloads.items(w)
    si = oracle.SortedItems(items, w.V)
    for _ in range(args.warmup):
        oracle_decode_sample(w, items, si, [0], args.scores)
    secs, cands = 0.0, 0
    for i in range(args.steps):   # each step: the whole batch, as the GPU arm
        t, c = oracle_decode_sample(w, items, si, list(range(w.B)), args.scores)
        secs += t
        cands += c
    value = cands / secs
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": workload_config(w, args.scores),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"each step: full {w.S}-step decode of all {w.B} requests"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm

def algorithmic(w, s, logits_mode, nnz_step):
    """Required bytes / flops of the attention and the selection of step s >= 1."""
    B, BW, Hq, Hkv, D, V = w.B, w.BW, w.Hq, w.Hkv, w.D, w.V
    P = sum(int(x) for x in __import__("workloads").prompt_lengths(w)) / w.n_shared
    att_bytes = (2 * B * Hkv * P * D * 2            # shared K,V read once per request
                 + 2 * B * BW * Hkv * s * D * 2     # distinct earlier unshared tokens
                 + 2 * B * BW * Hkv * D * 2 * 2     # this step's k/v: read + append
                 + 2 * B * BW * Hq * D * 2          # q read + O write
                 + B * BW * Hq * 4)                 # LSE
    att_flops = 4.0 * B * BW * Hq * D * (P + s + 1)
    sel_bytes = (B * BW * V * 4 if logits_mode else nnz_step * 4) + nnz_step * 4 + B * BW * 16
    return att_bytes, att_flops, sel_bytes


def attention_bw512(dev, hbm, tf, src, reps=5):
    """The metric's second half, "attention HBM GB/s vs peak (BW=512)": the staged
    attention of the 512x512 candidate pool (gr-decode-pool-512x512: 32 requests,
    4096-token prompts, 512 beams, Hq 32 / Hkv 8) at step 1, with the step's mask
    built beside it as in the decode.  One graph of the phase, replayed with the
    L2 flushed before each replay (the phase rewrites the same outputs and the
    same Unshared slots, so every replay does the same work); required bytes
    (shared KV once per request, the beams' Unshared tokens, this step's k/v
    read and appended, q, O, LSE) per median replay time."""
    import torch
    import workloads
    from shared_prefix_decode_xattention_b200 import xgr
    from shared_prefix_decode_xattention_b200.session import Session, config_for
    w = workloads.WORKLOADS[3]
    items = workloads.items(w)
    sess = Session(config_for(w), dev)
    sess.build_trie(items)
    for r in range(w.B):
        k, v = workloads.shared_kv(w, w.shared_id(r), dev)
        sess.prefill(r, w.shared_id(r), k, v)
    del k, v
    qkv = [workloads.step_qkv(w, s, dev) for s in range(2)]
    out = torch.empty((w.B, w.BW, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.BW, w.Hq), dtype=torch.float32, device=dev)
    par = torch.empty((w.B, w.BW), dtype=torch.int32, device=dev)
    tok = torch.empty_like(par)
    cum = torch.empty((w.B, w.BW), dtype=torch.float32, device=dev)
    nout = torch.empty((w.B,), dtype=torch.int32, device=dev)
    cur = torch.cuda.current_stream
    side = torch.cuda.Stream(device=dev)
    sess.begin(w.B, cur())
    sc0 = workloads.step_logits(w, 0, dev)
    m0 = sess.build_mask(0, cur())
    sess.decode_step(0, *qkv[0], out, lse, cur())
    sess.beam_select(0, sc0, xgr.XGR_SCORES_LOGITS, m0, par, tok, cum, nout, cur())
    torch.cuda.synchronize()
    del sc0
    keep = []

    def phase():
        side.wait_stream(cur())
        with torch.cuda.stream(side):
            keep.append(sess.build_mask(1, side))
        sess.decode_step(1, *qkv[1], out, lse, cur())
        cur().wait_stream(side)

    phase()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        phase()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        flush.zero_()
        g.replay()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    status = sess.device_status()
    del g
    sess.close()
    ms = statistics.median(ts)
    att_bytes, att_flops, _ = algorithmic(w, 1, True, 0)
    gbs = att_bytes / (ms / 1e3) / 1e9
    tfl = att_flops / (ms / 1e3) / 1e12
    return {"workload": f"{w.name}: B={w.B}, prompt {w.prompt[0]} tokens, BW={w.BW}, "
                        f"Hq={w.Hq}, Hkv={w.Hkv}, D={w.D}, step 1 (mask built beside it)",
            "ms": ms, "required_bytes": att_bytes, "achieved_gbs": gbs, "peak_gbs": hbm,
            "frac": gbs / hbm, "tflops": tfl, "tensor_peak_tflops": tf, "tensor_frac": tfl / tf,
            "peak_source": src, "l2": "flushed before each of the timed replays",
            "kernel": attention_kernel(w),
            "traffic": measured_traffic(attention_kernel(w), w.name),
            "device_status": status}


def _timed_graph(fn, dev, reps=5, warm=3):
    """Median device time (ms) of one CUDA graph of fn, replayed with the L2
    flushed (a 256 MiB write) before every replay."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(warm):
        flush.zero_()
        g.replay()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    del g
    return statistics.median(ts)


def per_beam_baseline(dev, hbm, src):
    """The pages' kernel-level comparison (xGR page, 1 "Problem definition" and 4
    "Kernel efficiency"): one decode step of the 128x128-pool workload through
    the staged attention (xgr_decode_step) and through the per-beam path
    (xgr_decode_step_per_beam: every beam reads its whole prompt and copies its
    parent's token block on the fork), on the same beam state (step 1, after a
    real step-0 selection), each replayed as a graph with the L2 flushed."""
    import torch
    import workloads
    from shared_prefix_decode_xattention_b200 import xgr
    from shared_prefix_decode_xattention_b200.session import Session, config_for
    w = workloads.WORKLOADS[2]
    sess = Session(config_for(w), dev)
    sess.build_trie(workloads.items(w))
    for r in range(w.B):
        k, v = workloads.shared_kv(w, w.shared_id(r), dev)
        sess.prefill(r, w.shared_id(r), k, v)
    cur = torch.cuda.current_stream
    out = torch.empty((w.B, w.BW, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.BW, w.Hq), dtype=torch.float32, device=dev)
    par = torch.empty((w.B, w.BW), dtype=torch.int32, device=dev)
    tok, cum = torch.empty_like(par), torch.empty((w.B, w.BW), dtype=torch.float32, device=dev)
    nout = torch.empty((w.B,), dtype=torch.int32, device=dev)
    sess.begin(w.B, cur())
    q0, k0, v0 = workloads.step_qkv(w, 0, dev)
    sess.decode_step(0, q0, k0, v0, out, lse, cur())            # the pool's step-0 tokens
    sess.decode_step_per_beam(0, q0, k0, v0, out, lse, cur())   # the blocks' step-0 tokens
    sess.beam_select(0, workloads.step_logits(w, 0, dev), xgr.XGR_SCORES_LOGITS, sess.build_mask(0),
                     par, tok, cum, nout, cur())
    q1, k1, v1 = workloads.step_qkv(w, 1, dev)
    staged = _timed_graph(lambda: sess.decode_step(1, q1, k1, v1, out, lse, cur()), dev)
    beam = _timed_graph(lambda: sess.decode_step_per_beam(1, q1, k1, v1, out, lse, cur()), dev)
    status = sess.device_status()
    sess.close()
    P = int(workloads.prompt_lengths(w)[0])
    units = w.B * w.BW * w.Hkv
    # per (request, beam, kv head): its whole prompt and its 2 own tokens (K and V),
    # the parent's 16-token block copied (read + write) and this step's token
    per_beam_bytes = units * (2 * (P + 2) * w.D * 2 + 2 * 2 * 16 * w.D * 2)
    return {"workload": f"{w.name}: B={w.B}, prompt {P}, BW={w.BW}, Hq={w.Hq}, Hkv={w.Hkv}, D={w.D}, step 1",
            "staged_attention_ms": staged, "per_beam_ms": beam,
            "per_beam_over_staged": beam / staged,
            "per_beam_bytes_moved": per_beam_bytes,
            "per_beam_gbs": per_beam_bytes / (beam / 1e3) / 1e9,
            # what any per-beam kernel needs to move its bytes at the copy bandwidth,
            # over the staged step: a ratio that does not depend on this baseline's tuning
            "per_beam_bytes_at_copy_bw_ms": per_beam_bytes / hbm / 1e6,
            "bound_ratio_at_copy_bw": per_beam_bytes / hbm / 1e6 / staged,
            "note": "a straightforward CUDA-core per-beam kernel (eight warps per (request, beam, kv head)); "
                    "its prompt re-reads are mostly L2 hits (a request's prompt is 2 MB)",
            "context": "xGR page, 4 Kernel efficiency: about 6.6x lower kernel latency than PagedAttention "
                       "(their hardware)",
            "peak_gbs": hbm, "peak_source": src, "device_status": status}


def prefix_batches(dev, hbm, tf, src):
    """Feather's comparison (Feather page, "Results": prefix-homogeneous batches
    against heterogeneous ones), kernel side: the staged attention of the
    prefix-shared workload (64 requests, beam 1, 8192-token prefixes shared in 4
    groups of 16, private suffixes of 256-2048 tokens) against the same request
    lengths with 64 distinct prefixes.  One decode step each, replayed as a graph
    with the L2 flushed; required bytes = every prefix and suffix K/V once, q, O,
    LSE, this step's k/v read and appended."""
    import torch
    import workloads
    from shared_prefix_decode_xattention_b200 import xgr
    from shared_prefix_decode_xattention_b200.session import Session, config_for
    out = {}
    for kind, w in (("homogeneous", workloads.WORKLOADS[4]),
                    ("heterogeneous", workloads.heterogeneous(workloads.WORKLOADS[4]))):
        sess = Session(config_for(w), dev)
        for sid in range(w.n_shared):
            members = [r for r in range(w.B) if w.shared_id(r) == sid]
            k, v = workloads.shared_kv(w, sid, dev)
            sess.prefill(members[0], sid, k, v)
            for r in members[1:]:
                sess.link(r, sid)
            del k, v
        for r in range(w.B):
            k, v = workloads.suffix_kv(w, r, dev)
            sess.prefill(r, 0, k, v, kind=xgr.XGR_KV_SUFFIX)
            del k, v
        q, kn, vn = workloads.step_qkv(w, 0, dev)
        o = torch.empty((w.B, w.BW, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.BW, w.Hq), dtype=torch.float32, device=dev)
        sess.begin(w.B)
        cur = torch.cuda.current_stream

        def step():
            sess.begin(w.B, cur())
            sess.decode_step(0, q, kn, vn, o, lse, cur())

        ms = _timed_graph(step, dev)
        status = sess.device_status()
        sess.close()
        kv_tok = int(workloads.prompt_lengths(w).sum()) + int(workloads.suffix_lengths(w).sum())
        req = (2 * w.Hkv * w.D * 2 * kv_tok + 2 * w.B * w.Hkv * w.D * 2 * 2
               + 2 * w.B * w.Hq * w.D * 2 + w.B * w.Hq * 4)
        gbs = req / (ms / 1e3) / 1e9
        keys = sum(int(workloads.prompt_lengths(w)[w.shared_id(r)]) + int(workloads.suffix_lengths(w)[r]) + 1
                   for r in range(w.B))
        tfl = 4.0 * w.Hq * w.D * keys / (ms / 1e3) / 1e12
        out[kind] = {"ms": ms, "required_bytes": req, "achieved_gbs": gbs, "frac": gbs / hbm,
                     "tflops": tfl, "device_status": status}
    out["time_ratio_heterogeneous_over_homogeneous"] = (out["heterogeneous"]["ms"]
                                                         / out["homogeneous"]["ms"])
    out["context"] = ("Feather reports about 2x throughput for homogeneous batches with unmodified "
                      "kernels on A100 / RTX 6000 Ada (Feather page, Results)")
    out["peak_gbs"] = hbm
    out["peak_source"] = src
    out["workload"] = ("prefix-shared-llm-decode: 64 requests, beam 1, 8192-token prefixes in 4 groups "
                       "of 16 (heterogeneous: 64 distinct), suffixes 256-2048, Hq=32, Hkv=8, D=128")
    return out


def batch_formation(dev, src, batch=16, chunk=256):
    """Feather's batching on the kernel side (Feather page, "Methodology", 1.
    Chunked Hash Tree, and "Results"): the 64 requests of the prefix-shared
    workload (4 prompt families of 16; 8192-token family prefixes, private
    suffixes of 256-2048 tokens) arrive in a shuffled order.  The batches the
    tree forms from their token ids are timed against batches of 16 consecutive
    arrivals.  A batch is one context: each family it holds is one shared KV
    segment (loaded once, linked by the batch's other members of that family),
    each request adds its suffix; one decode step per batch, one graph each,
    the L2 flushed before each; the figure is the sum over the batches."""
    import numpy as np
    import torch
    import workloads
    from shared_prefix_decode_xattention_b200 import xgr
    from shared_prefix_decode_xattention_b200.sched import ChunkedHashTree
    from shared_prefix_decode_xattention_b200.session import Session
    w = workloads.WORKLOADS[4]
    lens, suf = workloads.prompt_lengths(w), workloads.suffix_lengths(w)
    rng = np.random.default_rng(4242)
    fam = [rng.integers(0, 32000, size=int(lens[g])) for g in range(w.n_shared)]
    toks = [np.concatenate([fam[w.shared_id(r)], rng.integers(0, 32000, size=int(suf[r]))])
            for r in range(w.B)]
    arrivals = [int(r) for r in np.random.default_rng(7).permutation(w.B)]
    tree = ChunkedHashTree(chunk)
    for r in arrivals:
        tree.insert(r, toks[r])
    formed = tree.form_batches(batch, 1)
    tree.close()
    for members, shared in formed:   # each batch shares its family's whole prefix
        if shared * chunk != int(lens[w.shared_id(members[0])]):
            raise RuntimeError("the tree's batches do not share their whole prefix")
    batchings = (("tree", [list(m) for m, _ in formed]),
                 ("arrival_order", [arrivals[i:i + batch] for i in range(0, w.B, batch)]))
    q, kn, vn = workloads.step_qkv(w, 0, dev)
    fam_kv = {g: workloads.shared_kv(w, g, dev) for g in range(w.n_shared)}
    cur = torch.cuda.current_stream
    out = {}
    for kind, batches in batchings:
        ms = 0.0
        n_prefix = 0
        status = 0
        for members in batches:
            n = len(members)
            fams = sorted({w.shared_id(r) for r in members})
            kv_tokens = sum(int(lens[g]) for g in fams) + sum(int(suf[r]) for r in members)
            cfg = xgr.make_config(max_requests=n, max_shared=len(fams), kv_tokens=kv_tokens,
                                  beam_width=1, top_k=1, steps=1, n_q_heads=w.Hq, n_kv_heads=w.Hkv,
                                  head_dim=w.D, vocab=0, max_items=0, max_fanout=0, max_partials=0)
            sess = Session(cfg, dev)
            for sid, g in enumerate(fams):
                idx = [i for i, r in enumerate(members) if w.shared_id(r) == g]
                sess.prefill(idx[0], sid, *fam_kv[g])
                for i in idx[1:]:
                    sess.link(i, sid)
            for i, r in enumerate(members):
                k, v = workloads.suffix_kv(w, r, dev)
                sess.prefill(i, 0, k, v, kind=xgr.XGR_KV_SUFFIX)
            sel = torch.tensor(members, device=dev)
            qb, knb, vnb = q[sel].contiguous(), kn[sel].contiguous(), vn[sel].contiguous()
            o = torch.empty((n, 1, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
            lse = torch.empty((n, 1, w.Hq), dtype=torch.float32, device=dev)
            sess.begin(n)

            def step():
                sess.begin(n, cur())
                sess.decode_step(0, qb, knb, vnb, o, lse, cur())

            ms += _timed_graph(step, dev)
            status |= sess.device_status()
            sess.close()
            n_prefix += len(fams)
        prefix_bytes = n_prefix * 2 * w.Hkv * int(lens[0]) * w.D * 2
        out[kind] = {"ms": ms, "batches": len(batches), "prefix_segments": n_prefix,
                     "prefix_bytes_read": prefix_bytes, "device_status": status}
    out["time_ratio_arrival_over_tree"] = out["arrival_order"]["ms"] / out["tree"]["ms"]
    out["workload"] = ("prefix-shared-llm-decode: 64 requests in a shuffled arrival order, batches of 16: "
                       "Chunked Hash Tree (256-token chunks) against consecutive arrivals")
    out["context"] = ("Feather reports about 2x throughput for homogeneous batches (Feather page, Results); "
                      "here arrival-order batches still share a prefix among their members of one family")
    out["peak_source"] = src
    return out


def long_history(dev, hbm, tf, src, reps=3):
    """The long-history ragged workload (128 requests, prompts of 2048-16384
    tokens, 256 beams, Hq 32 / Hkv 4, D 128, V 16384, logits) at step 1: the
    staged attention (its mask built beside it) and the selection, each timed
    between events around its own graph, after a graph that replays the decode
    up to that step; the L2 is flushed before every repetition."""
    import torch
    import workloads
    from shared_prefix_decode_xattention_b200 import xgr
    from shared_prefix_decode_xattention_b200.session import Session, config_for
    w = workloads.WORKLOADS[5]
    items = workloads.items(w)
    sess = Session(config_for(w), dev)
    sess.build_trie(items)
    del items
    for r in range(w.B):
        k, v = workloads.shared_kv(w, w.shared_id(r), dev)
        sess.prefill(r, w.shared_id(r), k, v)
        del k, v
    qkv = [workloads.step_qkv(w, s, dev) for s in range(2)]
    sc = [workloads.step_logits(w, s, dev) for s in range(2)]
    o = torch.empty((w.B, w.BW, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.BW, w.Hq), dtype=torch.float32, device=dev)
    par = torch.empty((w.B, w.BW), dtype=torch.int32, device=dev)
    tok = torch.empty_like(par)
    cum = torch.empty((w.B, w.BW), dtype=torch.float32, device=dev)
    nout = torch.empty((w.B,), dtype=torch.int32, device=dev)
    cur = torch.cuda.current_stream
    side = torch.cuda.Stream(device=dev)
    masks = {}
    F = xgr.XGR_SCORES_LOGITS

    def head():
        sess.begin(w.B, cur())
        masks[0] = sess.build_mask(0, cur())
        sess.decode_step(0, *qkv[0], o, lse, cur())
        sess.beam_select(0, sc[0], F, masks[0], par, tok, cum, nout, cur())

    def att():
        side.wait_stream(cur())
        with torch.cuda.stream(side):
            masks[1] = sess.build_mask(1, side)
        sess.decode_step(1, *qkv[1], o, lse, cur())
        cur().wait_stream(side)

    def sel():
        sess.beam_select(1, sc[1], F, masks[1], par, tok, cum, nout, cur())

    head()
    att()
    torch.cuda.synchronize()
    nnz = sess.mask_entries(masks[1])
    sel()
    torch.cuda.synchronize()
    graphs = []
    for fn in (head, att, sel):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        graphs.append(g)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    att_ms, sel_ms = [], []
    for i in range(reps + 1):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        graphs[0].replay()
        ev[0].record()
        graphs[1].replay()
        ev[1].record()
        graphs[2].replay()
        ev[2].record()
        torch.cuda.synchronize()
        if i:
            att_ms.append(ev[0].elapsed_time(ev[1]))
            sel_ms.append(ev[1].elapsed_time(ev[2]))
    status = sess.device_status()
    del graphs
    sess.close()
    att_bytes, att_flops, sel_bytes = algorithmic(w, 1, True, nnz)
    am, sm = statistics.median(att_ms), statistics.median(sel_ms)
    return {"workload": f"{w.name}: B={w.B}, prompts {w.prompt[0]}-{w.prompt[1]} tokens, BW={w.BW}, "
                        f"Hq={w.Hq}, Hkv={w.Hkv}, D={w.D}, V={w.V}, step 1, logits",
            "attention_ms": am, "attention_required_bytes": att_bytes,
            "attention_gbs": att_bytes / (am / 1e3) / 1e9,
            "attention_hbm_frac": att_bytes / (am / 1e3) / 1e9 / hbm,
            "attention_tflops": att_flops / (am / 1e3) / 1e12,
            "attention_tensor_frac": att_flops / (am / 1e3) / 1e12 / tf,
            "select_ms": sm, "select_required_bytes": sel_bytes,
            "select_gbs": sel_bytes / (sm / 1e3) / 1e9,
            "select_hbm_frac": sel_bytes / (sm / 1e3) / 1e9 / hbm,
            "csr_entries_step1": nnz, "peak_gbs": hbm, "tensor_peak_tflops": tf,
            "peak_source": src, "l2": "flushed before each repetition", "device_status": status}


def max_over_ranks(x: float, device) -> float:
    """The largest value over all ranks (one all-reduce; the value itself with one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def decode_required_bytes(w, logits_mode, nnz):
    """Bytes one decode must move at least: per step, every prompt and suffix
    K/V once, each live beam's earlier Unshared k/v, this step's k/v (read and
    appended), q and O and LSE, the score rows the selection needs (full rows
    of the live beams with logits, the masked entries with log-probs), the
    mask (bitset, or CSR row pointers + entries + the trie tokens copied) and
    the selection's outputs."""
    B, BW, Hq, Hkv, D, V = w.B, w.BW, w.Hq, w.Hkv, w.D, w.V
    import workloads
    kv_tokens = int(workloads.prompt_lengths(w).sum()) + int(workloads.suffix_lengths(w).sum())
    shared = 2 * Hkv * D * 2 * kv_tokens          # every prompt / suffix K and V once per step
    total = 0
    for s in range(w.S):
        live = B * (1 if (s == 0 and V) else BW)
        b = shared
        b += 2 * live * Hkv * s * D * 2            # earlier Unshared k/v
        b += 2 * live * Hkv * D * 2 * 2            # this step's k/v: read + append
        b += 2 * live * Hq * D * 2 + live * Hq * 4  # q, O, LSE
        if V:
            if s == 0:
                b += B * V * 4 + (V + 7) // 8      # beam 0's score row, bitset
            else:
                b += (live * V * 4 if logits_mode else nnz[s] * 4)
                b += (B * BW + 1) * 4 + nnz[s] * 4 * 2   # row_ptr, cols written, trie tokens read
            b += B * BW * 16                       # parent, token, cum, n_out
        total += b
    return total


def code_sha(path: str) -> str:
    """SHA-256 of a CUDA/C++ source with its comments and whitespace removed:
    the code the counters were taken on, unchanged by edits of comments."""
    import hashlib
    import re
    text = open(path, encoding="utf-8").read()
    text = re.sub(r"//[^\n]*|/\*.*?\*/", " ", text, flags=re.S)
    return hashlib.sha256(" ".join(text.split()).encode()).hexdigest()


def measured_traffic(call: str, workload: str):
    """DRAM bytes per launch of a call on a workload, from the committed ncu
    summary (profiles/traffic.json), or None when there is no capture of that
    call on that workload or the code of any of the call's kernel sources has
    changed since the counters were taken (code_sha differs)."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))[call]
        if rec.get("workload_name") != workload:
            return None
        for rel, sha in rec["sources"].items():
            if code_sha(os.path.join(ROOT, rel)) != sha:
                return None
        return rec["dram_bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        return None


def _pct(xs, q):
    """The q-th percentile of sorted values (nearest rank)."""
    if not xs:
        return None
    return xs[min(len(xs) - 1, max(0, int(round(q / 100 * (len(xs) - 1)))))]


def secondary_rates(w, items, nnz, ms):
    """The step's other throughputs: valid (beam, token) candidates scored per
    second (step 0: one live beam per request against the distinct first
    tokens; later steps: the mask's measured entries) and vocabulary entries
    scored per second (live beams x V; logits mode reads every one)."""
    import numpy as np
    first = int(np.unique(items[:, 0]).size) * w.B
    valid = first + sum(nnz[1:])
    scored = sum(w.B * (1 if s == 0 else w.BW) * w.V for s in range(w.S))
    return {"valid_candidates_per_s": valid / (ms / 1e3), "tokens_scored_per_s": scored / (ms / 1e3),
            "valid_candidates_per_decode": valid, "tokens_scored_per_decode": scored}


def attention_kernel(w):
    """The attention kernel the work plan runs at steps >= 1 for a workload of
    single-request segments: the tensor-core one (D = 128), in its one-O
    variant when no item passes 12 key chunks, else the small-row kernel with
    the merge."""
    if w.D != 128:
        return "attn_small_kernel + attn_merge_kernel"
    return "attn_tc_one_o_kernel" if -(-w.prompt[1] // 128) <= 12 else "attn_tc_kernel"


def run_gpu(args, w):
    import numpy as np
    import torch
    import torch.distributed as dist

    import workloads
    from shared_prefix_decode_xattention_b200 import xgr
    from shared_prefix_decode_xattention_b200.session import Session, config_for

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(dev))

    # weak scaling: rank r decodes its own B requests (shard r of the batch)
    w = workloads.shard_of(w, rank)
    items = workloads.items(w)
    logits_mode = args.scores == "logits"
    flags = xgr.XGR_SCORES_LOGITS if logits_mode else xgr.XGR_SCORES_LOGPROB
    # Request groups: the batch split into G contexts whose decodes run on G
    # streams of one graph (requests are independent; one group's selection
    # overlaps another's attention -- the multi-stream batching of the xGR
    # page's xSchedule, applied to the hot path).  G = 1: one context.
    G = max(1, min(args.groups, w.B))
    while w.B % G:
        G -= 1
    Bg = w.B // G
    wg = workloads.small(w, B=Bg)   # the shape of one group's context
    sessions = []
    for g in range(G):
        sg = Session(config_for(wg), dev)
        sg.build_trie(items)
        for i in range(Bg):
            r = g * Bg + i
            k, v = workloads.shared_kv(w, w.shared_id(r), dev)
            sg.prefill(i, i, k, v)
        sessions.append(sg)
    del k, v
    inputs = []
    for s in range(w.S):
        q, kn, vn = workloads.step_qkv(w, s, dev)
        sc = (workloads.step_logits if logits_mode else workloads.step_logprobs)(w, s, dev)
        inputs.append((q, kn, vn, sc))
    out = torch.empty((w.B, w.BW, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.BW, w.Hq), dtype=torch.float32, device=dev)
    par = torch.empty((w.B, w.BW), dtype=torch.int32, device=dev)
    tok = torch.empty_like(par)
    cum = torch.empty((w.B, w.BW), dtype=torch.float32, device=dev)
    # one n_out per group (the call wants 16-byte aligned outputs; a group's
    # slice of one [B] array is not when B / G is not a multiple of 4)
    nout_g = [torch.empty((Bg,), dtype=torch.int32, device=dev) for _ in range(G)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for sg in sessions:
        sg.begin(Bg)   # plan once (setup)
    torch.cuda.synchronize()

    ev = lambda: torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream
    streams = [torch.cuda.Stream(device=dev) for _ in range(G)]
    sl = lambda g: slice(g * Bg, (g + 1) * Bg)

    # One decode = phases: [begin + step 0] then, for s >= 1, [attention s] and
    # [mask + selection s].  Each phase is enqueued on the current stream (the
    # capture stream while a CUDA graph is recorded), forked into one stream
    # per request group and joined again; with `host`, the step's inputs come
    # from pinned host memory and its outputs go back to it.  The masks are
    # views (xgr_build_mask enqueues nothing).
    masks = [[None] * w.S for _ in range(G)]

    def fork(body):
        top = cur()
        for g in range(G):
            streams[g].wait_stream(top)
            with torch.cuda.stream(streams[g]):
                body(g, streams[g])
        for g in range(G):
            top.wait_stream(streams[g])

    def att_g(g, st, s, inp, host):
        q, kn, vn, sc = inp[s]
        masks[g][s] = sessions[g].build_mask(s, st)
        if host is not None:
            for d, h in zip(inp[s], host[s]):
                d[sl(g)].copy_(h[sl(g)], non_blocking=True)
        sessions[g].decode_step(s, q[sl(g)], kn[sl(g)], vn[sl(g)], out[sl(g)], lse[sl(g)], st)

    def sel_g(g, st, s, inp, host):
        sessions[g].beam_select(s, inp[s][3][sl(g)], flags, masks[g][s], par[sl(g)], tok[sl(g)],
                                cum[sl(g)], nout_g[g], st)
        if host is not None:
            for h, d in zip(host[w.S + s], (par, tok, cum)):
                h[sl(g)].copy_(d[sl(g)], non_blocking=True)
            host[w.S + s][3][sl(g)].copy_(nout_g[g], non_blocking=True)

    def enqueue_att(s, inp, host):
        fork(lambda g, st: att_g(g, st, s, inp, host))

    def enqueue_sel(s, inp, host):
        fork(lambda g, st: sel_g(g, st, s, inp, host))

    def head_g(g, st, inp, host):
        sessions[g].begin(Bg, st)
        att_g(g, st, 0, inp, host)
        sel_g(g, st, 0, inp, host)

    def enqueue_head(inp, host):
        fork(lambda g, st: head_g(g, st, inp, host))

    def enqueue_decode(inp=inputs, host=None):
        def chain(g, st):   # a group's whole decode on its own stream
            head_g(g, st, inp, host)
            for s in range(1, w.S):
                att_g(g, st, s, inp, host)
                sel_g(g, st, s, inp, host)
        fork(chain)

    def capture(fn, keep=False):
        g = torch.cuda.CUDAGraph(keep_graph=keep)
        with torch.cuda.graph(g):
            fn()
        if keep:
            g.instantiate()
        return g

    for _ in range(max(args.warmup, 3)):   # eager warm-up (plans, attributes)
        enqueue_decode()
    torch.cuda.synchronize()
    # valid (row, token) entries of every step (one eager decode, summed over groups)
    nnz = [0] * w.S
    for g in range(G):
        sessions[g].begin(Bg, cur())
    for s in range(w.S):
        enqueue_att(s, inputs, None)
        torch.cuda.synchronize()
        for g in range(G):
            m = masks[g][s]
            nnz[s] += sessions[g].mask_entries(m) if m.kind != xgr.XGR_MASK_DENSE else 0
        enqueue_sel(s, inputs, None)
    torch.cuda.synchronize()
    if any(sg.device_status() != 0 for sg in sessions):
        raise RuntimeError("device status set during warm-up")
    # the graph-based execution of the pages' system level: a whole decode is one
    # graph, built by the library (xgr_decode_graph_create), each request group's
    # chain on its own stream
    decode_graph = xgr.xgr_decode_graph_create(
        [dict(ctx=sessions[g].ctx, n_requests=Bg, score_flags=flags,
              q=[inputs[s][0][sl(g)] for s in range(w.S)], k_new=[inputs[s][1][sl(g)] for s in range(w.S)],
              v_new=[inputs[s][2][sl(g)] for s in range(w.S)], scores=[inputs[s][3][sl(g)] for s in range(w.S)],
              out=out[sl(g)], lse=lse[sl(g)], parent=par[sl(g)], token=tok[sl(g)], cum=cum[sl(g)],
              n_out=nout_g[g]) for g in range(G)], w.S)
    launches_per_decode = xgr.xgr_decode_graph_kernels(decode_graph)
    g_phase = [capture(lambda: enqueue_head(inputs, None))]
    for s in range(1, w.S):
        g_phase.append(capture(lambda s=s: enqueue_att(s, inputs, None)))
        g_phase.append(capture(lambda s=s: enqueue_sel(s, inputs, None)))
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        xgr.xgr_decode_graph_launch(decode_graph, cur())
    torch.cuda.synchronize()

    # ---- timed region: K whole-decode graph replays, L2 flushed before each
    starts, ends = [ev() for _ in range(args.steps)], [ev() for _ in range(args.steps)]
    clk = Clocks(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record()
        xgr.xgr_decode_graph_launch(decode_graph, cur())
        ends[i].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = clk.stop() if clk else None
    step_ms = sorted(a.elapsed_time(b) for a, b in zip(starts, ends))
    total_ms = max_over_ranks(sum(step_ms), dev)
    n_live = torch.cat(nout_g).cpu().numpy()
    cands = candidates_per_decode(w) * args.steps * world
    value = cands / (total_ms / 1e3)

    # ---- per-phase device time (same decode, one graph per phase, events between)
    att_ms, sel_ms = [], []
    for i in range(args.steps):
        flush.zero_()
        evs = [ev() for _ in range(len(g_phase) + 1)]
        evs[0].record()
        for k, g in enumerate(g_phase):
            g.replay()
            evs[k + 1].record()
        torch.cuda.synchronize()
        for k in range(1, len(g_phase)):
            (att_ms if k % 2 == 1 else sel_ms).append(evs[k].elapsed_time(evs[k + 1]))

    # ---- end to end through the C ABI with host buffers (copies inside the graph)
    e2e = None
    if not args.no_e2e:
        host = []
        h2d = d2h = 0
        for s in range(w.S):
            hs = [t.cpu().pin_memory() for t in inputs[s]]
            host.append(hs)
            h2d += sum(t.numel() * t.element_size() for t in hs)
        for s in range(w.S):
            hs = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (par, tok, cum)]
            hs.append(torch.empty((w.B,), dtype=torch.int32).pin_memory())
            host.append(hs)
            d2h += sum(t.numel() * t.element_size() for t in hs)
        dev_in = [tuple(torch.empty_like(t) for t in inputs[s]) for s in range(w.S)]
        enqueue_decode(dev_in, host)
        torch.cuda.synchronize()
        g_e2e = capture(lambda: enqueue_decode(dev_in, host))
        g_e2e.replay()
        torch.cuda.synchronize()
        e_s, e_e = [ev() for _ in range(args.steps)], [ev() for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            e_s[i].record()
            g_e2e.replay()
            e_e[i].record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(e_s, e_e)), dev)
        e2e = {"value": cands / (e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}
        del g_e2e

    status = 0
    for sg in sessions:
        status |= sg.device_status()

    # ---- roofline of the dominant call (attention vs selection at steps >= 1)
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        pass
    hbm = peaks.get("hbm_gbs", 6650.0)
    tf = peaks.get("bf16_tflops", 1590.0)
    src = "of measured" if peaks else "of fallback"
    nnz_step = nnz[1] if w.S > 1 else 0   # CSR entries of step 1 (measured above)
    att_bytes, att_flops, sel_bytes = algorithmic(w, 1, logits_mode, nnz_step)
    required = decode_required_bytes(w, logits_mode, nnz)
    dec_gbs = required / (total_ms / args.steps / 1e3) / 1e9
    att_avg = statistics.mean(att_ms) / 1e3
    sel_avg = statistics.mean(sel_ms) / 1e3
    # the dominant kernel (largest share of the decode in the ncu launch list,
    # profiles/launches_*.md): the tensor-core attention, one launch per step --
    # for short items (workload 2: 8 prompt chunks + 1) the one-O variant
    # attn_tc_one_o_kernel -- timed by its phase graph (the attention of a step
    # is that one launch)
    achieved = att_flops / att_avg / 1e12
    att_kernel = attention_kernel(w)
    roof = {"kernel": f"{att_kernel} (xgr_decode_step, steps >= 1)", "bound": "tensor",
            "achieved": achieved, "peak": tf, "unit": "TFLOP/s", "frac": achieved / tf,
            "peak_source": f"bf16_tflops burst {src}",
            "traffic": measured_traffic(att_kernel, w.name),
            "algorithmic_per_launch": att_flops, "launch_ms": att_avg * 1e3,
            "hbm_gbs_required_bytes": att_bytes / att_avg / 1e9,
            "hbm_frac_required_bytes": att_bytes / att_avg / 1e9 / hbm}
    # the selection call (select_rows_kernel + select_pick_kernel) against HBM
    sel_gbs = sel_bytes / sel_avg / 1e9
    select_call = {"call": "xgr_beam_select (steps >= 1: select_rows_kernel, select_pick_kernel)",
                   "bound": "hbm", "achieved": sel_gbs, "peak": hbm, "unit": "GB/s",
                   "frac": sel_gbs / hbm, "algorithmic_per_call": sel_bytes,
                   "call_ms": sel_avg * 1e3,
                   "traffic_rows_kernel": measured_traffic("select_rows_kernel", w.name)}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, args.scores),
            "global_batch": w.B * world, "parallelism": f"dp{world}" if world > 1 else "single",
            "roofline": roof,
            "select_call": select_call,
            "step_breakdown_ms": {"attention_with_mask_step_ge1": att_avg * 1e3,
                                  "select_step_ge1": sel_avg * 1e3},
            "decode_hbm": {"required_bytes_per_decode": required, "achieved_gbs": dec_gbs,
                           "peak_gbs": hbm, "frac": dec_gbs / hbm,
                           "note": "whole decode (all steps, every kernel) against the copy "
                                   f"bandwidth {src}"},
            "step_ms_percentiles": {"p10": _pct(step_ms, 10), "p50": _pct(step_ms, 50),
                                    "p90": _pct(step_ms, 90), "replays": len(step_ms),
                                    "note": "this rank's timed replays"},
            "secondary_rates": secondary_rates(w, items, nnz, total_ms / args.steps),
            "request_groups": G,
            "gpu_launches": launches_per_decode * args.steps,
            "device_status": status, "n_live_last": int(n_live.min()) if n_live.size else 0}
    if e2e:
        line["e2e"] = e2e
    if clocks:
        line["clocks"] = clocks
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, items, args.scores)
    xgr.xgr_decode_graph_destroy(decode_graph)
    del g_phase   # released before the next workload's session
    if world == 1 and not args.no_bw512:
        line["attention_bw512"] = attention_bw512(dev, hbm, tf, src)
    if world == 1 and not args.no_extra:
        line["per_beam_baseline"] = per_beam_baseline(dev, hbm, src)
        line["prefix_batches"] = prefix_batches(dev, hbm, tf, src)
        line["batch_formation"] = batch_formation(dev, src)
        line["long_history"] = long_history(dev, hbm, tf, src)
    # the Shared stage's tensor throughput per workload (the stage is a dense
    # contraction; its tensor fraction is what bounds it at 128+ beams)
    tfr = {f"{w.name} (step >= 1, with the Unshared and Merging stages)": att_flops / att_avg / 1e12 / tf}
    if "attention_bw512" in line:
        tfr["gr-decode-pool-512x512 (step 1)"] = line["attention_bw512"]["tensor_frac"]
    if "long_history" in line:
        tfr["long-history-ragged-gr-decode (step 1)"] = line["long_history"]["attention_tensor_frac"]
    if "prefix_batches" in line:
        tfr["prefix-shared-llm-decode homogeneous"] = line["prefix_batches"]["homogeneous"]["tflops"] / tf
    line["shared_stage_tensor_frac"] = tfr
    if rank == 0:
        print(json.dumps(line), flush=True)
    for sg in sessions:
        sg.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    import workloads
    w = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()

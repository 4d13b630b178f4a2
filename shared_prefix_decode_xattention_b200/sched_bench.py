"""Host cost of forming prefix-homogeneous batches with the Chunked Hash Tree.

    python -m shared_prefix_decode_xattention_b200.sched_bench [--requests N]
        [--groups G] [--prefix P] [--suffix-max S] [--chunk C] [--max-batch M]

Seeded synthetic requests: G groups sharing P-token prefixes, each request with
its own 0..S-token suffix, arriving in random order.  Prints one JSON line:
the time to insert them (hashing included), to form every batch with the
static policy, and the per-decision cost (one decision per request added).
"""
from __future__ import annotations

import argparse
import json
import time

import numpy as np

from .sched import ChunkedHashTree


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--requests", type=int, default=20000)
    ap.add_argument("--groups", type=int, default=100)
    ap.add_argument("--prefix", type=int, default=8192)
    ap.add_argument("--suffix-max", type=int, default=2048)
    ap.add_argument("--chunk", type=int, default=256)
    ap.add_argument("--max-batch", type=int, default=256)
    a = ap.parse_args()
    rng = np.random.default_rng(1)
    prefixes = [rng.integers(0, 32000, size=a.prefix, dtype=np.int32) for _ in range(a.groups)]
    group = rng.integers(0, a.groups, size=a.requests)
    prompts = [np.concatenate([prefixes[g], rng.integers(0, 32000, size=int(rng.integers(0, a.suffix_max + 1)),
                                                         dtype=np.int32)]) for g in group]
    tokens = sum(len(p) for p in prompts)
    t = ChunkedHashTree(a.chunk)
    t0 = time.perf_counter()
    for i, p in enumerate(prompts):
        t.insert(i, p)
    t1 = time.perf_counter()
    batches = t.form_batches(a.max_batch, max(1, a.prefix // a.chunk // 2))
    t2 = time.perf_counter()
    print(json.dumps({
        "requests": a.requests, "groups": a.groups, "chunk_tokens": a.chunk, "prompt_tokens": tokens,
        "insert_s": t1 - t0, "insert_mtokens_per_s": tokens / (t1 - t0) / 1e6,
        "form_s": t2 - t1, "batches": len(batches),
        "us_per_decision": (t2 - t1) / a.requests * 1e6,
    }))


if __name__ == "__main__":
    main()

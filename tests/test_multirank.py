"""The multi-GPU path on CPU: two gloo ranks, as bench.py runs under torchrun.

The decode shards by request (each GPU takes B requests of the batch, no
exchange on the data path); the only collective is the max over ranks of the
timed region.  Checked here without a GPU:
  * every rank draws its own requests (prompts, queries, scores) but the same
    global item set;
  * bench.max_over_ranks returns the largest value of all ranks;
  * each rank's oracle decode of its shard yields only valid items, and the
    union over ranks holds as many decodes as requests in the batch.
"""
import hashlib
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _digest(a) -> int:
    return int(hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()[:15], 16)


def _rank(rank: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        import bench
        import oracle

        base = workloads.WORKLOADS[1]
        w = workloads.shard_of(base, rank)
        # the rank's own requests, one global item set
        mine = torch.tensor([_digest(workloads.step_logits(w, 0, "cpu").numpy()),
                             _digest(workloads.step_qkv(w, 0, "cpu")[0].view(torch.int16).numpy()),
                             _digest(workloads.shared_kv(w, 0, "cpu")[0].view(torch.int16).numpy()),
                             _digest(workloads.items(w))], dtype=torch.int64)
        every = [torch.zeros_like(mine) for _ in range(WORLD)]
        dist.all_gather(every, mine)
        # the timed region: the slowest rank decides
        t_max = bench.max_over_ranks(1.5 + rank, "cpu")
        # the rank's shard decodes to valid items (oracle, tiny workload)
        items = workloads.items(w)
        item_set = {tuple(x) for x in items.tolist()}
        si = oracle.SortedItems(items, w.V)
        n_valid = 0
        for r in range(w.B):
            dec = oracle.BeamDecode(si, w.BW, w.K, w.S, w.Hq, w.Hkv, w.D, w.V, mode="logprob")
            dec.begin(*_prompt(w, r))
            for s in range(w.S):
                q, kn, vn = workloads.step_qkv(w, s, "cpu")
                dec.attention(s, q[r], kn[r], vn[r])
                lp = workloads.step_logprobs(w, s, "cpu").numpy()[r]
                dec.select(s, lp, dec.mask(s))
            n_valid += sum(tuple(p) in item_set for p in dec.paths[:dec.n_live].tolist())
        counts = torch.tensor([w.B, n_valid], dtype=torch.int64)
        dist.all_reduce(counts)
        out[rank] = (torch.stack(every).tolist(), t_max, counts.tolist())
    finally:
        dist.destroy_process_group()


def _prompt(w, r):
    k, v = workloads.shared_kv(w, w.shared_id(r), "cpu")
    return k.view(torch.int16).numpy().view(np.uint16), v.view(torch.int16).numpy().view(np.uint16)


def test_two_ranks_shard_requests_and_reduce_time():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(port, out), nprocs=WORLD, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    every, t0, counts = res[0]
    assert res[1][0] == every                      # both ranks saw the same gather
    logits, q, prompt, item_hash = zip(*every)
    assert logits[0] != logits[1] and q[0] != q[1] and prompt[0] != prompt[1]
    assert item_hash[0] == item_hash[1]            # the global item set
    assert t0 == res[1][1] == 2.5                  # max over ranks
    w = workloads.WORKLOADS[1]
    assert counts[0] == WORLD * w.B
    assert counts[1] == WORLD * w.B * min(w.BW, w.n_items)   # every live beam ends on an item

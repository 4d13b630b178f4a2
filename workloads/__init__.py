"""Seeded synthetic inputs for the beam-decode hot path.

This module only draws random numbers and fixes shapes.  It holds none of the
method's arithmetic (no attention, no masking, no selection), so both the CPU
oracle (``oracle/``) and the CUDA path read exactly the same inputs from it
while sharing no code with each other.

The five workloads follow the workload shapes of the xGR page ("xGR: Efficient
Generative Recommendation Serving at Scale", section 1 "Problem definition":
long user-history prompts, short fixed-length outputs, large beam width with
candidate pools such as 128x128 and 512x512) and of the Feather page ("Requests
of the same feather must flock together", "Results": batches that share 1K-10K
token prefixes).  The public datasets named there are not available, so these
synthetic draws stand in for them.

Seeds: every tensor is drawn from ``seed = 1000 * workload_id + tensor_id`` so
that any slice can be regenerated independently.  Large tensors are drawn with
torch's generator on the requested device (Philox on CUDA); the item set is
drawn on the host with numpy's PCG64.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

# tensor ids inside one workload's seed space
_T_ITEMS = 1
_T_PROMPT_LEN = 2
_T_SHARED_K = 3
_T_SHARED_V = 4
_T_SUFFIX_K = 5
_T_SUFFIX_V = 6
_T_SUFFIX_LEN = 7
_T_Q = 10
_T_KNEW = 20
_T_VNEW = 30
_T_LOGITS = 40


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one synthetic decode workload."""

    wid: int
    name: str
    B: int                      # requests in the batch
    prompt: tuple               # (min, max) prompt tokens, inclusive, uniform integers
    BW: int                     # beam width
    K: int                      # per-beam top-K
    S: int                      # decode steps == item length L
    Hq: int
    Hkv: int
    D: int
    V: int                      # tokens per level (0: no vocabulary / no selection)
    n_items: int                # distinct valid items (token tuples of length S)
    logits_std: float = 2.0     # "N(0,2)" read as standard deviation 2
    groups: int = 0             # >0: requests share prefixes in this many groups
    suffix: tuple = (0, 0)      # per-request unshared suffix length range (inclusive)
    shard: int = 0              # which B-request slice of a larger batch (one per GPU)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def n_shared(self) -> int:
        return self.groups if self.groups else self.B

    def shared_id(self, r: int) -> int:
        """Shared-prefix id of request r (contiguous groups of B/groups requests)."""
        if self.groups:
            return r // (self.B // self.groups)
        return r

    def candidates_per_step(self, s: int, n_live: Optional[int] = None) -> int:
        """Beam candidates scored at step s: B x live beams x K (the BW x K pool)."""
        n = 1 if s == 0 else self.BW if n_live is None else n_live
        return self.B * n * self.K


WORKLOADS = {
    1: Workload(1, "tiny-gr-beam-decode", B=1, prompt=(256, 256), BW=4, K=4, S=3,
                Hq=8, Hkv=2, D=64, V=256, n_items=1000),
    2: Workload(2, "gr-decode-pool-128x128", B=8, prompt=(1024, 1024), BW=128, K=128, S=3,
                Hq=16, Hkv=4, D=128, V=8192, n_items=1_000_000),
    3: Workload(3, "gr-decode-pool-512x512", B=32, prompt=(4096, 4096), BW=512, K=512, S=3,
                Hq=32, Hkv=8, D=128, V=8192, n_items=4_000_000),
    4: Workload(4, "prefix-shared-llm-decode", B=64, prompt=(8192, 8192), BW=1, K=1, S=1,
                Hq=32, Hkv=8, D=128, V=0, n_items=0, groups=4, suffix=(256, 2048)),
    5: Workload(5, "long-history-ragged-gr-decode", B=128, prompt=(2048, 16384), BW=256, K=256,
                S=4, Hq=32, Hkv=4, D=128, V=16384, n_items=8_000_000),
}


def heterogeneous(w: Workload) -> Workload:
    """The comparison run of the prefix-shared workload: every request its own prefix."""
    return dataclasses.replace(w, name=w.name + "-heterogeneous", groups=0)


def small(w: Workload, **kw) -> Workload:
    """A reduced copy of a workload (same distributions, smaller sizes) for fast tests."""
    return dataclasses.replace(w, **kw)


def shard_of(w: Workload, shard: int) -> Workload:
    """Requests shard*B .. shard*B + B-1 of a batch split over GPUs: the same shapes
    and the same global item set, their own prompts, queries and scores."""
    return dataclasses.replace(w, shard=shard)


def _seed(w: Workload, tid: int, extra: int = 0, per_shard: bool = True) -> int:
    return 1000 * w.wid + tid + 100_000 * extra + (10_000_000 * w.shard if per_shard else 0)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def items(w: Workload) -> np.ndarray:
    """Exactly ``n_items`` distinct S-token tuples drawn uniformly from [0, V)^S.

    Duplicates are rejected and redrawn; the result keeps first-draw order.
    Returns int32 [n_items][S].
    """
    rng = np.random.default_rng(_seed(w, _T_ITEMS, per_shard=False))   # one global item set
    n, L, V = w.n_items, w.S, w.V
    if n > V ** L:
        raise ValueError("more distinct items requested than tuples exist")
    out = np.empty((0, L), dtype=np.int64)
    seen = np.empty((0,), dtype=np.int64)
    while out.shape[0] < n:
        need = n - out.shape[0]
        draw = rng.integers(0, V, size=(need + need // 8 + 16, L), dtype=np.int64)
        code = np.zeros(draw.shape[0], dtype=np.int64)
        for j in range(L):
            code = code * V + draw[:, j]
        _, first = np.unique(code, return_index=True)
        first.sort()
        draw, code = draw[first], code[first]
        fresh = ~np.isin(code, seen)
        draw, code = draw[fresh][:need], code[fresh][:need]
        out = np.concatenate([out, draw])
        seen = np.concatenate([seen, code])
    return out.astype(np.int32)


def prompt_lengths(w: Workload) -> np.ndarray:
    """Prompt (shared prefix) length per shared id, uniform integers in ``w.prompt``."""
    lo, hi = w.prompt
    rng = np.random.default_rng(_seed(w, _T_PROMPT_LEN))
    return rng.integers(lo, hi + 1, size=w.n_shared).astype(np.int32)


def suffix_lengths(w: Workload) -> np.ndarray:
    """Per-request unshared suffix length (prefix-shared workload), uniform inclusive."""
    lo, hi = w.suffix
    if hi == 0:
        return np.zeros(w.B, dtype=np.int32)
    rng = np.random.default_rng(_seed(w, _T_SUFFIX_LEN))
    return rng.integers(lo, hi + 1, size=w.B).astype(np.int32)


def _bf16_normal(shape, seed, device):
    x = torch.randn(shape, generator=_gen(device, seed), device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def shared_kv(w: Workload, sid: int, device="cpu", length: Optional[int] = None):
    """Prompt K and V of shared id ``sid``: bf16 N(0,1), layout [Hkv][P][D]."""
    P = int(prompt_lengths(w)[sid]) if length is None else length
    k = _bf16_normal((w.Hkv, P, w.D), _seed(w, _T_SHARED_K, sid + 1), device)
    v = _bf16_normal((w.Hkv, P, w.D), _seed(w, _T_SHARED_V, sid + 1), device)
    return k, v


def suffix_kv(w: Workload, r: int, device="cpu"):
    """Per-request unshared suffix K and V: bf16 N(0,1), layout [Hkv][X][D]."""
    X = int(suffix_lengths(w)[r])
    k = _bf16_normal((w.Hkv, X, w.D), _seed(w, _T_SUFFIX_K, r + 1), device)
    v = _bf16_normal((w.Hkv, X, w.D), _seed(w, _T_SUFFIX_V, r + 1), device)
    return k, v


def step_qkv(w: Workload, s: int, device="cpu", copy: int = 0):
    """Fresh per-step tensors: q [B][BW][Hq][D], k_new, v_new [B][BW][Hkv][D], bf16 N(0,1).

    ``copy`` selects an independent redraw (used to rotate inputs between timed steps).
    """
    q = _bf16_normal((w.B, w.BW, w.Hq, w.D), _seed(w, _T_Q + s, copy), device)
    k = _bf16_normal((w.B, w.BW, w.Hkv, w.D), _seed(w, _T_KNEW + s, copy), device)
    v = _bf16_normal((w.B, w.BW, w.Hkv, w.D), _seed(w, _T_VNEW + s, copy), device)
    return q, k, v


def step_logits(w: Workload, s: int, device="cpu", copy: int = 0) -> torch.Tensor:
    """Per-step logits fp32 [B][BW][V], N(0, std=logits_std)."""
    x = torch.randn((w.B, w.BW, w.V), generator=_gen(device, _seed(w, _T_LOGITS + s, copy)),
                    device=device, dtype=torch.float32)
    return x * w.logits_std


def step_logprobs(w: Workload, s: int, device="cpu", copy: int = 0) -> torch.Tensor:
    """Per-step log-prob inputs fp32 [B][BW][V]: the logits above turned into
    full-vocabulary log-probabilities once, in fp64, then rounded to fp32.

    This is input synthesis (a realistic log-prob distribution); the selection
    under test receives these fp32 values as given on both sides.
    """
    x = step_logits(w, s, device, copy).double()
    return torch.log_softmax(x, dim=-1).float()

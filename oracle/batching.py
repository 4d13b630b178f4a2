"""Oracle of the prefix-homogeneous batch former -- TEST INFRASTRUCTURE.

Only ``tests/`` may import this module.  It shares no code with the library's
Chunked Hash Tree and uses no hashing at all: every quantity is recomputed from
the prompt tokens by direct comparison, the slow O(W x B x T) way the Feather
page contrasts the tree with.

Source: Feather page ("Requests of the same feather must flock together"),
"Methodology", 1. Chunked Hash Tree -- requests cut into fixed-size token
chunks; the batch being formed covers the chunks of its members; a waiting
request's missing count is the number of its chunks not covered; the best
request to add has the smallest missing count; the policy sees the batch size,
the loss of shared prefix depth (delta) and the number of waiting requests
that share the new depth (w), and adds the request or dispatches the batch.
The readings of what the page leaves open (full chunks only, the
earliest-inserted request seeding a batch and breaking ties, depth measured
against the first member, the static policy that adds the best request whose
depth stays at or above a floor and passes over the others) are the ones stated in the
library's header, restated here in terms of tokens.

Parity status: pinned by tests/test_sched_cht.py (a hand-derived example).
"""
from __future__ import annotations

from typing import Dict, List, Optional, Tuple


class BatchFormerOracle:
    def __init__(self, chunk: int):
        assert chunk >= 1
        self.C = chunk
        self.tokens: Dict[int, List[int]] = {}
        self.waiting: List[int] = []   # ids in insertion order
        self.batch: List[int] = []     # ids in join order

    # ---- definitions
    def chunks(self, r: int) -> int:
        """Full chunks of request r's prompt."""
        return len(self.tokens[r]) // self.C

    def shared(self, a: int, b: int) -> int:
        """Leading full chunks on which the prompts of a and b agree token for token."""
        ta, tb, C = self.tokens[a], self.tokens[b], self.C
        k = 0
        while k < min(self.chunks(a), self.chunks(b)) and ta[k * C:(k + 1) * C] == tb[k * C:(k + 1) * C]:
            k += 1
        return k

    def missing(self, r: int) -> int:
        """Chunks of r that no member of the batch also has (as a prefix)."""
        if not self.batch:
            return self.chunks(r)
        return self.chunks(r) - max(self.shared(r, m) for m in self.batch)

    def tip(self) -> int:
        """Leading chunks every member of the batch shares."""
        if not self.batch:
            return 0
        f = self.batch[0]
        return min(self.shared(m, f) if m != f else self.chunks(f) for m in self.batch)

    # ---- operations
    def insert(self, r: int, tokens) -> None:
        assert r not in self.tokens
        self.tokens[r] = [int(x) for x in tokens]
        self.waiting.append(r)

    def remove(self, r: int) -> None:
        self.waiting.remove(r)
        del self.tokens[r]

    def find_best(self) -> Optional[Tuple[int, int, int, int, int]]:
        """(id, missing, depth_after, delta, w) or None."""
        if not self.waiting:
            return None
        if not self.batch:
            r = self.waiting[0]
            d = self.chunks(r)
            ref, miss, delta = r, d, 0
        else:
            order = {q: i for i, q in enumerate(self.waiting)}
            r = min(self.waiting, key=lambda q: (self.missing(q), order[q]))
            ref = self.batch[0]
            d = min(self.tip(), self.shared(r, ref))
            miss, delta = self.missing(r), self.tip() - d
        w = 0
        if d > 0:
            for q in self.waiting:
                if q != r and self.chunks(q) >= d and self.shared(q, r) >= d:
                    w += 1
        return r, miss, d, delta, w

    def depth_after(self, r: int) -> int:
        """Chunks the batch would still share with r added: min(tip, shared with the first member)."""
        return min(self.tip(), self.shared(r, self.batch[0]))

    def best_passing(self, floor: int) -> Optional[int]:
        """The static policy's choice: among the waiting requests whose depth_after
        reaches the floor, the one with the smallest missing count, then the
        earliest inserted; None when none qualifies."""
        order = {q: i for i, q in enumerate(self.waiting)}
        ok = [q for q in self.waiting if self.depth_after(q) >= floor]
        if not ok:
            return None
        return min(ok, key=lambda q: (self.missing(q), order[q]))

    def add(self, r: int) -> None:
        self.waiting.remove(r)
        self.batch.append(r)

    def dispatch(self) -> Tuple[List[int], int]:
        out, sh = list(self.batch), self.tip()
        for m in self.batch:
            del self.tokens[m]
        self.batch = []
        return out, sh

    def form_batches(self, max_batch: int, min_shared_chunks: int) -> List[Tuple[List[int], int]]:
        res = []
        if self.batch:
            res.append(self.dispatch())
        while self.waiting:
            self.add(self.find_best()[0])   # the earliest-inserted request seeds the batch
            while len(self.batch) < max_batch:
                r = self.best_passing(min_shared_chunks)
                if r is None:
                    break
                self.add(r)
            res.append(self.dispatch())
        return res

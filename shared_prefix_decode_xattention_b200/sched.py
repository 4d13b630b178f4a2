"""Host-side batch former: the Chunked Hash Tree of ``include/xgr_sched.h``.

Argument marshalling only; the data structure and the batching loop run in
libxgr.so.  It groups waiting requests into prefix-homogeneous batches; each
batch is then one shared KV segment for the attention (``shared_id``).
"""
from __future__ import annotations

import ctypes
from typing import List, Optional, Tuple

import numpy as np

from . import xgr


class ChunkedHashTree:
    """One xgr_cht handle: chunk_tokens tokens per hashed chunk."""

    def __init__(self, chunk_tokens: int):
        self.h = ctypes.c_void_p()
        xgr._check("xgr_cht_create", xgr.lib().xgr_cht_create(chunk_tokens, ctypes.byref(self.h)))
        self.chunk_tokens = chunk_tokens

    def close(self):
        if self.h:
            xgr.lib().xgr_cht_destroy(self.h)
            self.h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def insert(self, request_id: int, tokens) -> None:
        t = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        ptr = t.ctypes.data_as(ctypes.c_void_p) if t.size else None
        xgr._check("xgr_cht_insert", xgr.lib().xgr_cht_insert(self.h, request_id, ptr, t.size))

    def remove(self, request_id: int) -> None:
        xgr._check("xgr_cht_remove", xgr.lib().xgr_cht_remove(self.h, request_id))

    def find_best(self) -> Optional[Tuple[int, int, int, int, int]]:
        """(request_id, missing, depth_after, delta, w) of the best waiting
        request for the batch being formed, or None when none waits."""
        rid = ctypes.c_int64()
        m, d, dl, w = (ctypes.c_int32() for _ in range(4))
        xgr._check("xgr_cht_find_best", xgr.lib().xgr_cht_find_best(
            self.h, ctypes.byref(rid), ctypes.byref(m), ctypes.byref(d), ctypes.byref(dl),
            ctypes.byref(w)))
        if rid.value < 0:
            return None
        return rid.value, m.value, d.value, dl.value, w.value

    def add(self, request_id: int) -> None:
        xgr._check("xgr_cht_add_to_batch", xgr.lib().xgr_cht_add_to_batch(self.h, request_id))

    def counts(self) -> Tuple[int, int]:
        """(waiting, in_batch)."""
        w, b = ctypes.c_int32(), ctypes.c_int32()
        xgr._check("xgr_cht_counts", xgr.lib().xgr_cht_counts(self.h, ctypes.byref(w), ctypes.byref(b)))
        return w.value, b.value

    def dispatch(self) -> Tuple[List[int], int]:
        """Closes the batch being formed: (member ids in join order, shared chunks)."""
        cap = max(1, self.counts()[1])
        ids = np.zeros(cap, dtype=np.int64)
        n, sh = ctypes.c_int32(), ctypes.c_int32()
        xgr._check("xgr_cht_dispatch", xgr.lib().xgr_cht_dispatch(
            self.h, ids.ctypes.data_as(ctypes.c_void_p), cap, ctypes.byref(n), ctypes.byref(sh)))
        return ids[:n.value].tolist(), sh.value

    def form_batches(self, max_batch: int, min_shared_chunks: int) -> List[Tuple[List[int], int]]:
        """Every waiting request into batches by the static policy: a list of
        (member ids in join order, shared chunks), in dispatch order."""
        w, b = self.counts()
        total = w + b
        cap_b = max(1, w + (1 if b else 0))
        ids = np.zeros(max(1, total), dtype=np.int64)
        sizes = np.zeros(cap_b, dtype=np.int32)
        shared = np.zeros(cap_b, dtype=np.int32)
        nb = ctypes.c_int32()
        vp = lambda a: a.ctypes.data_as(ctypes.c_void_p)
        xgr._check("xgr_cht_form_batches", xgr.lib().xgr_cht_form_batches(
            self.h, max_batch, min_shared_chunks, vp(ids), ids.size, vp(sizes), vp(shared), cap_b,
            ctypes.byref(nb)))
        out, at = [], 0
        for k in range(nb.value):
            out.append((ids[at:at + sizes[k]].tolist(), int(shared[k])))
            at += int(sizes[k])
        return out

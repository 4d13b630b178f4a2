"""Thin ctypes binding of libxgr.so (the C ABI declared in include/xgr.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  Device buffers may be passed as torch tensors (their
data_ptr() is used) or as integer addresses; streams as torch.cuda.Stream or
integer handles (0 = the legacy default stream).  A missing or unloadable
library raises at once -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import glob
import os
import re
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libxgr.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "xgr.h")

XGR_OK = 0
XGR_ERR_ARG = -1
XGR_ERR_SHAPE = -2
XGR_ERR_CAPACITY = -3
XGR_ERR_STATE = -4
XGR_ERR_CUDA = -5
XGR_ERR_DEVICE = -6
XGR_ERR_UNIMPLEMENTED = -7

XGR_DEV_NAN = 1
XGR_DEV_INDEX = 2
XGR_DEV_MASK = 4
XGR_DEV_CAPACITY = 8
XGR_DEV_TIMEOUT = 16

XGR_SCORES_LOGPROB = 0
XGR_SCORES_LOGITS = 1
XGR_KV_SHARED = 0
XGR_KV_SUFFIX = 1
XGR_MASK_DENSE = 0
XGR_MASK_CSR = 1
XGR_MASK_NODE_BITS = 2
XGR_MASK_TRIE_ROWS = 3


class XgrError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status} ({xgr_status_string(status)})")
        self.status = status


class xgr_config(ctypes.Structure):
    _fields_ = [
        ("max_requests", ctypes.c_int32),
        ("max_shared", ctypes.c_int32),
        ("kv_tokens", ctypes.c_int64),
        ("beam_width", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("steps", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("vocab", ctypes.c_int32),
        ("max_items", ctypes.c_int64),
        ("max_fanout", ctypes.c_int32),
        ("max_partials", ctypes.c_int32),
    ]


class xgr_mask(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("step", ctypes.c_int32),
        ("bits", ctypes.c_void_p),
        ("n_words", ctypes.c_int32),
        ("n_rows", ctypes.c_int32),
        ("row_ptr", ctypes.c_void_p),
        ("cols", ctypes.c_void_p),
        ("cols_capacity", ctypes.c_int64),
        ("row_node", ctypes.c_void_p),
        ("node_ptr", ctypes.c_void_p),
        ("n_nodes", ctypes.c_int32),
        ("row_stride", ctypes.c_int32),
    ]


class xgr_decode_group(ctypes.Structure):
    _fields_ = [
        ("ctx", ctypes.c_void_p),
        ("n_requests", ctypes.c_int32),
        ("score_flags", ctypes.c_int32),
        ("d_q", ctypes.POINTER(ctypes.c_void_p)),
        ("d_k_new", ctypes.POINTER(ctypes.c_void_p)),
        ("d_v_new", ctypes.POINTER(ctypes.c_void_p)),
        ("d_scores", ctypes.POINTER(ctypes.c_void_p)),
        ("d_out", ctypes.c_void_p),
        ("d_lse", ctypes.c_void_p),
        ("d_parent", ctypes.c_void_p),
        ("d_token", ctypes.c_void_p),
        ("d_cum", ctypes.c_void_p),
        ("d_n_out", ctypes.c_void_p),
    ]


_lib = None


def declared_functions() -> list:
    """Names of the entry points the headers in include/ declare."""
    names = set()
    for h in sorted(glob.glob(os.path.join(os.path.dirname(HEADER), "*.h"))):
        names |= set(re.findall(r"^\s*(?:xgr_status|const char \*|[a-z_]+)\s*\*?\s*(xgr_\w+)\s*\(",
                                open(h).read(), flags=re.M))
    return sorted(names)


def lib():
    """Load libxgr.so (built in-tree by build.py); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libxgr.so is not built ({LIB_PATH}); run "
                           "shared_prefix_decode_xattention_b200.build.build()")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    sig = {
        "xgr_workspace_bytes": [ctypes.POINTER(xgr_config), ctypes.POINTER(ctypes.c_size_t)],
        "xgr_create": [ctypes.POINTER(xgr_config), P, ctypes.c_size_t, ctypes.POINTER(P)],
        "xgr_destroy": [P],
        "xgr_build_trie": [P, P, i64, i32],
        "xgr_prefill_kv": [P, i32, i32, P, P, i32, i32, P],
        "xgr_reset_kv": [P],
        "xgr_begin": [P, i32, P],
        "xgr_decode_step": [P, i32, P, P, P, P, P, P],
        "xgr_per_beam_bytes": [P, ctypes.POINTER(ctypes.c_size_t)],
        "xgr_decode_step_per_beam": [P, i32, P, P, P, P, P, P, ctypes.c_size_t, P],
        "xgr_build_mask": [P, i32, ctypes.POINTER(xgr_mask), P],
        "xgr_mask_to_csr": [P, ctypes.POINTER(xgr_mask), P, P, i64, P],
        "xgr_beam_select": [P, i32, P, i32, ctypes.POINTER(xgr_mask), P, P, P, P, P],
        "xgr_get_sequences": [P, P, P],
        "xgr_device_status": [P, P, ctypes.POINTER(i32)],
        "xgr_beam_topk_noalloc": [i32, i32, i32, i32, P, i32, P, P, P, P, P, P, P, P, P, P],
        "xgr_decode_graph_create": [ctypes.POINTER(xgr_decode_group), i32, i32, ctypes.POINTER(P)],
        "xgr_decode_graph_launch": [P, P],
        "xgr_decode_graph_kernels": [P, ctypes.POINTER(i32)],
        "xgr_decode_graph_destroy": [P],
        # host-side batch former (include/xgr_sched.h)
        "xgr_cht_create": [i32, ctypes.POINTER(P)],
        "xgr_cht_destroy": [P],
        "xgr_cht_insert": [P, i64, P, i64],
        "xgr_cht_remove": [P, i64],
        "xgr_cht_find_best": [P, ctypes.POINTER(i64), ctypes.POINTER(i32), ctypes.POINTER(i32),
                              ctypes.POINTER(i32), ctypes.POINTER(i32)],
        "xgr_cht_add_to_batch": [P, i64],
        "xgr_cht_dispatch": [P, P, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)],
        "xgr_cht_counts": [P, ctypes.POINTER(i32), ctypes.POINTER(i32)],
        "xgr_cht_form_batches": [P, i32, i32, P, i64, P, P, i32, ctypes.POINTER(i32)],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = i32
    L.xgr_status_string.argtypes = [i32]
    L.xgr_status_string.restype = ctypes.c_char_p
    _lib = L
    return L


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn: str, st: int):
    if st != XGR_OK:
        raise XgrError(fn, st)


def xgr_status_string(status: int) -> str:
    return lib().xgr_status_string(status).decode()


def xgr_workspace_bytes(cfg: xgr_config) -> int:
    n = ctypes.c_size_t(0)
    _check("xgr_workspace_bytes", lib().xgr_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def xgr_create(cfg: xgr_config, workspace, nbytes: int) -> int:
    h = ctypes.c_void_p(0)
    _check("xgr_create", lib().xgr_create(ctypes.byref(cfg), _ptr(workspace), nbytes,
                                          ctypes.byref(h)))
    return h.value


def xgr_destroy(ctx: int) -> None:
    _check("xgr_destroy", lib().xgr_destroy(ctx))


def xgr_build_trie(ctx: int, items: np.ndarray) -> None:
    items = np.ascontiguousarray(items, dtype=np.int32)
    _check("xgr_build_trie", lib().xgr_build_trie(ctx, items.ctypes.data, items.shape[0],
                                                  items.shape[1]))


def xgr_prefill_kv(ctx: int, request: int, shared_id: int, k, v, length: int, kind: int,
                   stream=None) -> None:
    _check("xgr_prefill_kv", lib().xgr_prefill_kv(ctx, request, shared_id, _ptr(k), _ptr(v),
                                                  length, kind, _stream(stream)))


def xgr_reset_kv(ctx: int) -> None:
    _check("xgr_reset_kv", lib().xgr_reset_kv(ctx))


def xgr_begin(ctx: int, n_requests: int, stream=None) -> None:
    _check("xgr_begin", lib().xgr_begin(ctx, n_requests, _stream(stream)))


def xgr_decode_step(ctx: int, step: int, q, k_new, v_new, out, lse, stream=None) -> None:
    _check("xgr_decode_step", lib().xgr_decode_step(ctx, step, _ptr(q), _ptr(k_new), _ptr(v_new),
                                                    _ptr(out), _ptr(lse), _stream(stream)))


def xgr_per_beam_bytes(ctx: int) -> int:
    n = ctypes.c_size_t(0)
    _check("xgr_per_beam_bytes", lib().xgr_per_beam_bytes(ctx, ctypes.byref(n)))
    return n.value


def xgr_decode_step_per_beam(ctx: int, step: int, q, k_new, v_new, out, lse, blocks, nbytes: int,
                             stream=None) -> None:
    _check("xgr_decode_step_per_beam",
           lib().xgr_decode_step_per_beam(ctx, step, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out),
                                          _ptr(lse), _ptr(blocks), nbytes, _stream(stream)))


def xgr_build_mask(ctx: int, step: int, stream=None) -> xgr_mask:
    m = xgr_mask()
    _check("xgr_build_mask", lib().xgr_build_mask(ctx, step, ctypes.byref(m), _stream(stream)))
    return m


def xgr_mask_to_csr(ctx: int, mask: xgr_mask, row_ptr, cols, cols_capacity: int, stream=None) -> None:
    _check("xgr_mask_to_csr", lib().xgr_mask_to_csr(ctx, ctypes.byref(mask), _ptr(row_ptr), _ptr(cols),
                                                    cols_capacity, _stream(stream)))


def xgr_beam_select(ctx: int, step: int, scores, flags: int, mask: xgr_mask, parent, token, cum,
                    n_out, stream=None) -> None:
    _check("xgr_beam_select", lib().xgr_beam_select(ctx, step, _ptr(scores), flags,
                                                    ctypes.byref(mask), _ptr(parent), _ptr(token),
                                                    _ptr(cum), _ptr(n_out), _stream(stream)))


def xgr_get_sequences(ctx: int, seq, stream=None) -> None:
    _check("xgr_get_sequences", lib().xgr_get_sequences(ctx, _ptr(seq), _stream(stream)))


def xgr_device_status(ctx: int, stream=None) -> int:
    """Synchronise, return the device status word (0 = clean) and clear it."""
    code = ctypes.c_int32(0)
    st = lib().xgr_device_status(ctx, _stream(stream), ctypes.byref(code))
    if st not in (XGR_OK, XGR_ERR_DEVICE):
        raise XgrError("xgr_device_status", st)
    return code.value


def xgr_beam_topk_noalloc(n_requests: int, beam_width: int, top_k: int, vocab: int, scores,
                          flags: int, cum, n_live, bits, row_ptr, cols, parent, token, cum_out,
                          n_out, stream=None) -> None:
    """Masked top-K without a context or any allocation (see include/xgr.h).

    Tensor arguments must be contiguous CUDA tensors of the types the header
    states (the call itself cannot see a host pointer or a wrong element size,
    and it reports no device status): scores, cum, cum_out fp32; n_live,
    row_ptr, cols, parent, token, n_out int32; bits int32 or uint32.  Integer
    addresses are passed through unchecked."""
    import torch
    want = {"scores": (scores, (torch.float32,)), "cum": (cum, (torch.float32,)),
            "n_live": (n_live, (torch.int32,)), "bits": (bits, (torch.int32, torch.uint32)),
            "row_ptr": (row_ptr, (torch.int32,)), "cols": (cols, (torch.int32,)),
            "parent": (parent, (torch.int32,)), "token": (token, (torch.int32,)),
            "cum_out": (cum_out, (torch.float32,)), "n_out": (n_out, (torch.int32,))}
    for name, (t, dtypes) in want.items():
        if t is None or isinstance(t, int):
            continue
        if not (t.is_cuda and t.is_contiguous() and t.dtype in dtypes):
            raise XgrError(f"xgr_beam_topk_noalloc({name}: {t.dtype}, "
                           f"{'cuda' if t.is_cuda else 'host'}, "
                           f"{'contiguous' if t.is_contiguous() else 'strided'})", XGR_ERR_ARG)
    _check("xgr_beam_topk_noalloc", lib().xgr_beam_topk_noalloc(
        n_requests, beam_width, top_k, vocab, _ptr(scores), flags, _ptr(cum), _ptr(n_live),
        _ptr(bits), _ptr(row_ptr), _ptr(cols), _ptr(parent), _ptr(token), _ptr(cum_out),
        _ptr(n_out), _stream(stream)))


def xgr_decode_graph_create(groups, steps: int) -> int:
    """The whole-decode graph of include/xgr.h.  `groups`: one dict per request
    group with keys ctx, n_requests, score_flags, q, k_new, v_new, scores
    (sequences of `steps` device buffers) and out, lse, parent, token, cum,
    n_out (device buffers).  Returns the graph handle."""
    n = len(groups)
    arr = (xgr_decode_group * max(n, 1))()
    keep = []
    for i, g in enumerate(groups):
        x = arr[i]
        x.ctx = g["ctx"]
        x.n_requests = g["n_requests"]
        x.score_flags = g["score_flags"]
        for field in ("q", "k_new", "v_new", "scores"):
            ptrs = (ctypes.c_void_p * max(1, len(g[field])))(*[_ptr(t) for t in g[field]])
            keep.append(ptrs)
            setattr(x, "d_" + field, ctypes.cast(ptrs, ctypes.POINTER(ctypes.c_void_p)))
        for field in ("out", "lse", "parent", "token", "cum", "n_out"):
            setattr(x, "d_" + field, _ptr(g[field]))
    h = ctypes.c_void_p(0)
    _check("xgr_decode_graph_create", lib().xgr_decode_graph_create(arr, n, steps, ctypes.byref(h)))
    return h.value


def xgr_decode_graph_launch(graph: int, stream=None) -> None:
    _check("xgr_decode_graph_launch", lib().xgr_decode_graph_launch(graph, _stream(stream)))


def xgr_decode_graph_kernels(graph: int) -> int:
    n = ctypes.c_int32(0)
    _check("xgr_decode_graph_kernels", lib().xgr_decode_graph_kernels(graph, ctypes.byref(n)))
    return n.value


def xgr_decode_graph_destroy(graph: int) -> None:
    _check("xgr_decode_graph_destroy", lib().xgr_decode_graph_destroy(graph))


def make_config(**kw) -> xgr_config:
    c = xgr_config()
    for k, v in kw.items():
        setattr(c, k, v)
    return c

"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/xgr.h declares, validates configurations, and fails
cleanly (no crash) when no CUDA device is present."""
import ctypes

import pytest
import torch

from shared_prefix_decode_xattention_b200 import build, xgr


@pytest.fixture(scope="module")
def L():
    build.build()
    return xgr.lib()


def test_every_declared_entry_point_is_exported(L):
    names = xgr.declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n


def _cfg(**kw):
    base = dict(max_requests=8, max_shared=8, kv_tokens=8192, beam_width=128, top_k=128,
                steps=3, n_q_heads=16, n_kv_heads=4, head_dim=128, vocab=8192,
                max_items=1_000_000)
    base.update(kw)
    return xgr.make_config(**base)


def test_mask_struct_matches_the_header(L):
    """xgr_mask as ctypes lays it out: the field order and the 72 bytes of the
    C struct (natural alignment on x86-64)."""
    names = [f[0] for f in xgr.xgr_mask._fields_]
    assert names == ["kind", "step", "bits", "n_words", "n_rows", "row_ptr", "cols",
                     "cols_capacity", "row_node", "node_ptr", "n_nodes", "row_stride"]
    assert ctypes.sizeof(xgr.xgr_mask) == 72


def test_workspace_bytes_for_a_valid_config(L):
    n = xgr.xgr_workspace_bytes(_cfg())
    assert n % 256 == 0 and n > 8192 * 4 * 128 * 2 * 2


@pytest.mark.parametrize("bad,status", [
    (dict(beam_width=0), xgr.XGR_ERR_SHAPE),
    (dict(top_k=64), xgr.XGR_ERR_SHAPE),                # K < BW
    (dict(n_q_heads=12, n_kv_heads=5), xgr.XGR_ERR_SHAPE),
    (dict(n_q_heads=48, n_kv_heads=4), xgr.XGR_ERR_UNIMPLEMENTED),   # G = 12
    (dict(head_dim=96), xgr.XGR_ERR_UNIMPLEMENTED),
    (dict(steps=9), xgr.XGR_ERR_SHAPE),
    (dict(vocab=-1), xgr.XGR_ERR_SHAPE),
    (dict(kv_tokens=1 << 31), xgr.XGR_ERR_SHAPE),
])
def test_invalid_configs_are_rejected(L, bad, status):
    with pytest.raises(xgr.XgrError) as e:
        xgr.xgr_workspace_bytes(_cfg(**bad))
    assert e.value.status == status


def test_null_arguments(L):
    assert L.xgr_workspace_bytes(None, None) == xgr.XGR_ERR_ARG
    assert L.xgr_destroy(None) == xgr.XGR_ERR_ARG
    assert L.xgr_begin(None, 1, None) == xgr.XGR_ERR_ARG
    assert L.xgr_decode_step(None, 0, None, None, None, None, None, None) == xgr.XGR_ERR_ARG
    m = xgr.xgr_mask()
    assert L.xgr_beam_select(None, 0, None, 0, ctypes.byref(m), None, None, None, None,
                             None) == xgr.XGR_ERR_ARG
    assert L.xgr_mask_to_csr(None, ctypes.byref(m), None, None, 1, None) == xgr.XGR_ERR_ARG
    assert xgr.xgr_status_string(xgr.XGR_ERR_CAPACITY).startswith("capacity")


def test_create_rejects_small_or_misaligned_workspace(L):
    cfg = _cfg()
    h = ctypes.c_void_p(0)
    assert L.xgr_create(ctypes.byref(cfg), 4096, 16, ctypes.byref(h)) == xgr.XGR_ERR_CAPACITY
    assert L.xgr_create(ctypes.byref(cfg), 4100, 1 << 40, ctypes.byref(h)) == xgr.XGR_ERR_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_create_without_a_device_fails_cleanly(L):
    cfg = _cfg()
    h = ctypes.c_void_p(0)
    n = xgr.xgr_workspace_bytes(cfg)
    assert L.xgr_create(ctypes.byref(cfg), 1 << 20, n, ctypes.byref(h)) == xgr.XGR_ERR_CUDA


def test_decode_group_struct_matches_the_header(L):
    """xgr_decode_group as ctypes lays it out: 13 fields, 96 bytes (natural
    alignment on x86-64: the pointer after the three 32-bit fields is padded to
    offset 24)."""
    names = [f[0] for f in xgr.xgr_decode_group._fields_]
    assert names == ["ctx", "n_requests", "score_flags", "d_q", "d_k_new", "d_v_new", "d_scores",
                     "d_out", "d_lse", "d_parent", "d_token", "d_cum", "d_n_out"]
    assert xgr.xgr_decode_group.d_q.offset == 16
    assert ctypes.sizeof(xgr.xgr_decode_group) == 96


def test_decode_graph_rejects_bad_arguments_before_any_device_work(L):
    h = ctypes.c_void_p(0)
    arr = (xgr.xgr_decode_group * 2)()
    assert L.xgr_decode_graph_create(None, 1, 3, ctypes.byref(h)) == xgr.XGR_ERR_ARG
    assert L.xgr_decode_graph_create(arr, 1, 3, None) == xgr.XGR_ERR_ARG
    assert L.xgr_decode_graph_create(arr, 1, 3, ctypes.byref(h)) == xgr.XGR_ERR_ARG   # NULL ctx
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the checks come first
    ptrs = (ctypes.c_void_p * 3)(1 << 20, 1 << 21, 1 << 22)
    for g in arr:
        g.ctx = fake
        for f in ("d_q", "d_k_new", "d_v_new", "d_scores"):
            setattr(g, f, ctypes.cast(ptrs, ctypes.POINTER(ctypes.c_void_p)))
    assert L.xgr_decode_graph_create(arr, 2, 3, ctypes.byref(h)) == xgr.XGR_ERR_ARG   # shared ctx
    assert L.xgr_decode_graph_create(arr, 0, 3, ctypes.byref(h)) == xgr.XGR_ERR_ARG
    assert L.xgr_decode_graph_create(arr, 65, 3, ctypes.byref(h)) == xgr.XGR_ERR_ARG
    assert L.xgr_decode_graph_create(arr, 1, 0, ctypes.byref(h)) == xgr.XGR_ERR_ARG
    arr[0].d_scores = None
    assert L.xgr_decode_graph_create(arr, 1, 3, ctypes.byref(h)) == xgr.XGR_ERR_ARG
    assert h.value is None
    n = ctypes.c_int32(0)
    assert L.xgr_decode_graph_launch(None, None) == xgr.XGR_ERR_ARG
    assert L.xgr_decode_graph_kernels(None, ctypes.byref(n)) == xgr.XGR_ERR_ARG
    assert L.xgr_decode_graph_destroy(None) == xgr.XGR_ERR_ARG

"""One libxgr context plus its device workspace (a convenience over ``xgr``).

PyTorch provides the device memory and the stream; every computation runs in
the library's kernels.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from . import xgr


class Session:
    """Owns a workspace tensor and an xgr_ctx on the current CUDA device."""

    def __init__(self, cfg: xgr.xgr_config, device: str = "cuda"):
        import torch
        self.cfg = cfg
        self.nbytes = xgr.xgr_workspace_bytes(cfg)
        # 256-byte alignment: torch's CUDA caching allocator returns 512-byte aligned blocks
        self.workspace = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        assert self.workspace.data_ptr() % 256 == 0
        self.ctx = xgr.xgr_create(cfg, self.workspace, self.nbytes)

    def close(self):
        if self.ctx:
            xgr.xgr_destroy(self.ctx)
            self.ctx = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # thin forwards -----------------------------------------------------------
    def build_trie(self, items: np.ndarray):
        xgr.xgr_build_trie(self.ctx, items)

    def prefill(self, request: int, shared_id: int, k, v, kind: int = xgr.XGR_KV_SHARED,
                stream=None):
        length = 0 if k is None else int(k.shape[1])
        xgr.xgr_prefill_kv(self.ctx, request, shared_id, k, v, length, kind, stream)

    def link(self, request: int, shared_id: int, stream=None):
        xgr.xgr_prefill_kv(self.ctx, request, shared_id, None, None, 0, xgr.XGR_KV_SHARED, stream)

    def begin(self, n_requests: int, stream=None):
        xgr.xgr_begin(self.ctx, n_requests, stream)

    def decode_step(self, step, q, k_new, v_new, out, lse, stream=None):
        xgr.xgr_decode_step(self.ctx, step, q, k_new, v_new, out, lse, stream)

    def decode_step_per_beam(self, step, q, k_new, v_new, out, lse, stream=None):
        """The per-beam comparison path (its private blocks allocated on first use)."""
        import torch
        if getattr(self, "_pb_blocks", None) is None:
            n = xgr.xgr_per_beam_bytes(self.ctx)
            self._pb_blocks = torch.zeros(n, dtype=torch.uint8, device=self.workspace.device)
        xgr.xgr_decode_step_per_beam(self.ctx, step, q, k_new, v_new, out, lse, self._pb_blocks,
                                     self._pb_blocks.numel(), stream)

    def build_mask(self, step, stream=None) -> xgr.xgr_mask:
        return xgr.xgr_build_mask(self.ctx, step, stream)

    def mask_csr(self, mask: xgr.xgr_mask, stream=None):
        """The rows of a step >= 1 mask as CSR device tensors (row_ptr int32
        [n_rows+1], cols int32 [cap]; the valid length is row_ptr[-1])."""
        import torch
        dev = self.workspace.device
        cap = max(1, mask.n_rows * max(1, mask.row_stride))
        row_ptr = torch.empty(mask.n_rows + 1, dtype=torch.int32, device=dev)
        cols = torch.empty(cap, dtype=torch.int32, device=dev)
        xgr.xgr_mask_to_csr(self.ctx, mask, row_ptr, cols, cap, stream)
        return row_ptr, cols

    def mask_entries(self, mask: xgr.xgr_mask) -> int:
        """Valid (row, token) entries of a step >= 1 mask (synchronises)."""
        import torch
        row_ptr, _ = self.mask_csr(mask)
        torch.cuda.synchronize()
        return int(row_ptr[-1].item())

    def beam_select(self, step, scores, flags, mask, parent, token, cum, n_out, stream=None):
        xgr.xgr_beam_select(self.ctx, step, scores, flags, mask, parent, token, cum, n_out, stream)

    def sequences(self, seq, stream=None):
        xgr.xgr_get_sequences(self.ctx, seq, stream)

    def device_status(self, stream=None) -> int:
        return xgr.xgr_device_status(self.ctx, stream)


def config_for(w, kv_tokens: Optional[int] = None, max_fanout: int = 0, max_items: int = 0,
               max_partials: int = 0) -> xgr.xgr_config:
    """xgr_config sized for a workload description (see workloads.Workload)."""
    if kv_tokens is None:
        kv_tokens = w.n_shared * w.prompt[1] + w.B * w.suffix[1]
    return xgr.make_config(max_requests=w.B, max_shared=w.n_shared, kv_tokens=kv_tokens,
                           beam_width=w.BW, top_k=w.K, steps=w.S, n_q_heads=w.Hq,
                           n_kv_heads=w.Hkv, head_dim=w.D, vocab=w.V,
                           max_items=max(max_items, w.n_items, 1 if w.V else 0),
                           max_fanout=max_fanout, max_partials=max_partials)

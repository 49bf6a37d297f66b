"""One trigger window of the LSA indexer path on one GPU: buffers plus the five C-ABI calls.

Allocation and call order only (PyTorch holds the device memory); every stage is a kernel
of liblsa.so.  Order of the stages follows the hyper.ai summary ("Method") and the blog
review's sections 3-3.2: project -> score/threshold/OR/compact -> fetch -> Lightning Top-k.
"""
from __future__ import annotations

import torch

from . import lsa


class IndexerPath:
    """Device buffers for one window of B sequences (ragged, total_S entries per layer)."""

    def __init__(self, L, B, d, r, n_h, d_I, tau, k, total_S, row_bytes, dtype, kdtype,
                 device="cuda", with_scores=False, with_mask=False):
        self.L, self.B, self.d, self.r, self.n_h, self.d_I = L, B, d, r, n_h, d_I
        self.tau, self.k, self.total_S, self.row_bytes = tau, k, int(total_S), row_bytes
        self.dtype, self.kdtype = dtype, kdtype
        dev = torch.device(device)
        T = self.total_S
        u8 = torch.uint8

        def ws(nbytes):
            return torch.empty(max(int(nbytes), 256), dtype=u8, device=dev)

        self.q = torch.empty((L, B, n_h, d_I), dtype=dtype, device=dev)
        self.w = torch.empty((L, B, n_h), dtype=torch.float32, device=dev)
        self.ws_proj = ws(lsa.lsa_project_workspace_size(L, B, d, r, n_h, d_I, dtype))
        self.idx = torch.empty(T, dtype=torch.int32, device=dev)
        self.count = torch.empty(B, dtype=torch.int32, device=dev)
        self.ws_score = ws(lsa.lsa_score_select_workspace_size(L, B, T))
        self.scores = torch.empty((L, T), dtype=torch.float32, device=dev) if with_scores else None
        self.mask = torch.empty(T, dtype=u8, device=dev) if with_mask else None
        self.hot_kv = torch.empty((T, row_bytes), dtype=u8, device=dev)
        # E4M3 keys are decoded to bf16 by the fetch (scales kept apart)
        hot_dt = torch.bfloat16 if kdtype == torch.float8_e4m3fn else kdtype
        self.hot_K = torch.empty((T, d_I), dtype=hot_dt, device=dev)
        self.hot_scale = torch.empty(T, dtype=torch.float32, device=dev) if kdtype == torch.float8_e4m3fn else None
        self.topk_idx = torch.empty((B, tau, k), dtype=torch.int32, device=dev)
        self.topk_score = torch.empty((B, tau, k), dtype=torch.float32, device=dev)
        self.ws_topk = ws(lsa.lsa_lightning_topk_workspace_size(B, tau, T, k))

    def project(self, h, W_dq, W_iuq, W_w, stream=None):
        lsa.lsa_project(h, W_dq, W_iuq, W_w, self.q, self.w, self.ws_proj, stream=stream)

    def select(self, K, k_scale, seq_offsets, threshold=0.5, q=None, w=None, stream=None):
        lsa.lsa_memindex_score_select(self.q if q is None else q, self.w if w is None else w, K, k_scale,
                                      seq_offsets, self.total_S, threshold, self.idx, self.count, self.ws_score,
                                      scores_out=self.scores, mask_out=self.mask, stream=stream)

    def fetch(self, seq_offsets, pool, K_sel, k_scale_sel, stream=None):
        lsa.lsa_fetch_gather(self.idx, self.count, seq_offsets, self.total_S, pool, self.hot_kv, K_sel, k_scale_sel,
                             self.hot_K, self.hot_scale, stream=stream)

    def topk(self, q_dec, w_dec, seq_offsets, stream=None):
        lsa.lsa_lightning_topk(q_dec, w_dec, self.hot_K, self.hot_scale, self.idx, self.count, seq_offsets,
                               self.total_S, self.k, self.topk_idx, self.ws_topk, topk_score=self.topk_score,
                               stream=stream)

    def run(self, h, W_dq, W_iuq, W_w, K, k_scale, seq_offsets, pool, q_dec, w_dec, sel_layer=0,
            threshold=0.5, stream=None):
        """The whole hot path for one trigger window."""
        self.project(h, W_dq, W_iuq, W_w, stream)
        self.select(K, k_scale, seq_offsets, threshold, stream=stream)
        self.fetch(seq_offsets, pool, K[sel_layer], None if k_scale is None else k_scale[sel_layer], stream)
        self.topk(q_dec, w_dec, seq_offsets, stream)

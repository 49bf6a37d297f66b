"""One trigger window of the LSA indexer path on one GPU: buffers plus the five C-ABI calls.

Allocation and call order only (PyTorch holds the device memory); every stage is a kernel
of liblsa.so.  Order of the stages follows the hyper.ai summary ("Method") and the blog
review's sections 3-3.2: project -> score/threshold/OR/compact -> fetch -> Lightning Top-k.
"""
from __future__ import annotations

from contextlib import contextmanager

import torch

from . import lsa


@contextmanager
def _stage(name):
    """NVTX range around a stage's launches (ncu --nvtx / nsys show the stage boundaries)."""
    torch.cuda.nvtx.range_push(name)
    try:
        yield
    finally:
        torch.cuda.nvtx.range_pop()


class IndexerPath:
    """Device buffers for one window of B sequences (ragged, total_S entries per layer)."""

    def __init__(self, L, B, d, r, n_h, d_I, tau, k, total_S, row_bytes, dtype, kdtype,
                 device="cuda", with_scores=False, with_mask=False, incremental=False):
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
        # the incremental row fetch of run(prev=...): workspace and the count of rows that crossed the link
        self.ws_incr = ws(lsa.lsa_fetch_incremental_workspace_size(B, T)) if incremental else None
        self.host_rows = torch.zeros(1, dtype=torch.int32, device=dev) if incremental else None
        # the host-link row gather of run(), at a higher priority than the caller's stream so that its
        # few fat CTAs are placed before the Top-k's persistent CTAs fill the SMs
        self._link = torch.cuda.Stream(device=dev, priority=-1)

    def project(self, h, W_dq, W_iuq, W_w, stream=None):
        lsa.lsa_project(h, W_dq, W_iuq, W_w, self.q, self.w, self.ws_proj, stream=stream)

    def select(self, K, k_scale, seq_offsets, threshold=0.5, q=None, w=None, stream=None):
        lsa.lsa_memindex_score_select(self.q if q is None else q, self.w if w is None else w, K, k_scale,
                                      seq_offsets, self.total_S, threshold, self.idx, self.count, self.ws_score,
                                      scores_out=self.scores, mask_out=self.mask, stream=stream)

    def fetch(self, seq_offsets, pool, K_sel, k_scale_sel, stream=None):
        """Rows and keys in one launch."""
        lsa.lsa_fetch_gather(self.idx, self.count, seq_offsets, self.total_S, pool, self.hot_kv, K_sel, k_scale_sel,
                             self.hot_K, self.hot_scale, stream=stream)

    def fetch_keys(self, seq_offsets, K_sel, k_scale_sel, stream=None):
        """The keys of the fetched entries only (device to device; the Top-k needs nothing else)."""
        lsa.lsa_fetch_gather(self.idx, self.count, seq_offsets, self.total_S, None, None, K_sel, k_scale_sel,
                             self.hot_K, self.hot_scale, stream=stream)

    def fetch_rows(self, seq_offsets, pool, stream=None):
        """The KV rows of the fetched entries only, over the host link."""
        lsa.lsa_fetch_gather(self.idx, self.count, seq_offsets, self.total_S, pool, self.hot_kv, stream=stream)

    def fetch_rows_incremental(self, seq_offsets, pool, prev, stream=None):
        """The KV rows of the fetched entries with the previous window's rows resident: rows that
        both windows fetched are copied on the device, only the others cross the host link.
        prev = (idx, count, seq_offsets, total_S, hot_kv) of the previous window."""
        p_idx, p_count, p_offs, p_T, p_hot = prev
        lsa.lsa_fetch_gather_incremental(self.idx, self.count, seq_offsets, self.total_S, p_idx, p_count, p_offs, p_T,
                                         p_hot, pool, self.hot_kv, self.ws_incr, host_rows_out=self.host_rows,
                                         stream=stream)

    def topk(self, q_dec, w_dec, seq_offsets, stream=None):
        lsa.lsa_lightning_topk(q_dec, w_dec, self.hot_K, self.hot_scale, self.idx, self.count, seq_offsets,
                               self.total_S, self.k, self.topk_idx, self.ws_topk, topk_score=self.topk_score,
                               stream=stream)

    def run(self, h, W_dq, W_iuq, W_w, K, k_scale, seq_offsets, pool, q_dec, w_dec, sel_layer=0,
            threshold=0.5, stream=None, events=None, prev=None):
        """The whole hot path for one trigger window.

        The KV rows cross the host link on a second stream while the keys are gathered and the
        Top-k runs on `stream` (the Top-k reads only the keys); `stream` waits for both before
        it returns, so work queued on it afterwards sees the whole window.  events: optional
        list of 7 timing events, recorded at the stage boundaries (start, after project, after
        select, after the keys, after the Top-k, after the rows (second stream), end).
        prev: the previous window's (idx, count, seq_offsets, total_S, hot_kv); the rows then come
        from the incremental fetch (the path must be built with incremental=True), and the
        previous hot buffer must stay untouched until `stream` has passed this window.
        """
        st = torch.cuda.current_stream() if stream is None else stream
        ev = events if events is not None else [None] * 7
        rec = lambda e, s: e.record(s) if e is not None else None
        rec(ev[0], st)
        with _stage("lsa.project"):
            self.project(h, W_dq, W_iuq, W_w, st)
        rec(ev[1], st)
        with _stage("lsa.score_select"):
            self.select(K, k_scale, seq_offsets, threshold, stream=st)
        rec(ev[2], st)
        selected = torch.cuda.Event()
        selected.record(st)
        self._link.wait_event(selected)
        with _stage("lsa.fetch_rows"):
            if prev is None:
                self.fetch_rows(seq_offsets, pool, self._link)
            else:
                self.fetch_rows_incremental(seq_offsets, pool, prev, self._link)
        rec(ev[5], self._link)
        rows_done = torch.cuda.Event()
        rows_done.record(self._link)
        with _stage("lsa.fetch_keys"):
            self.fetch_keys(seq_offsets, K[sel_layer], None if k_scale is None else k_scale[sel_layer], st)
        rec(ev[3], st)
        with _stage("lsa.lightning_topk"):
            self.topk(q_dec, w_dec, seq_offsets, st)
        rec(ev[4], st)
        st.wait_event(rows_done)
        rec(ev[6], st)

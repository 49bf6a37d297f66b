"""Python binding of liblsa.so (include/lsa.h): argument marshalling only.

Each function takes torch tensors, checks device/dtype/shape/contiguity, and passes raw
pointers to the C entry point of the same name; every step runs in the library's CUDA
kernels.  There is no CPU path: if liblsa.so is missing or fails to load, importing this
module raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblsa.so")

LSA_F32, LSA_BF16, LSA_FP8_E4M3 = 0, 1, 2
LSA_MAX_TOPK = 4096
_STATUS = {0: "LSA_OK", 1: "LSA_ERR_INVALID_ARG", 2: "LSA_ERR_UNSUPPORTED", 3: "LSA_ERR_CUDA",
           4: "LSA_ERR_DEVICE_CHECK", 5: "LSA_ERR_WORKSPACE"}
DTYPE_CODE = {torch.float32: LSA_F32, torch.bfloat16: LSA_BF16, torch.float8_e4m3fn: LSA_FP8_E4M3}

# every function declared in include/lsa.h
EXPORTS = ("lsa_last_error", "lsa_version", "lsa_launch_count", "lsa_check_device", "lsa_selftest_wait_timeout",
           "lsa_project_workspace_size", "lsa_project",
           "lsa_score_select_workspace_size", "lsa_memindex_score_select",
           "lsa_memindex_score_select_static",
           "lsa_fetch_gather", "lsa_fetch_incremental_workspace_size", "lsa_fetch_gather_incremental",
           "lsa_lightning_topk_workspace_size", "lsa_lightning_topk",
           "lsa_lightning_topk_step_workspace_size", "lsa_lightning_topk_step",
           "lsa_golden_labels_workspace_size", "lsa_golden_labels",
           "lsa_indexer_train_workspace_size", "lsa_indexer_train_step",
           "lsa_pool_alloc", "lsa_pool_free")


class LSAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run sparse_kv_cache_memoryindexer_b200/build.py "
                          "(or __graft_entry__.build())")
    lib = C.CDLL(LIB_PATH)
    P, I, I64, SZ, F = C.c_void_p, C.c_int, C.c_int64, C.c_size_t, C.c_float
    sig = {
        "lsa_last_error": (C.c_char_p, []),
        "lsa_version": (C.c_char_p, []),
        "lsa_launch_count": (C.c_uint64, []),
        "lsa_check_device": (I, [P]),
        "lsa_selftest_wait_timeout": (I, [P, P]),
        "lsa_project_workspace_size": (SZ, [I, I, I, I, I, I, I]),
        "lsa_project": (I, [P, P, P, P, I, I, I, I, I, I, I, P, P, P, SZ, P]),
        "lsa_score_select_workspace_size": (SZ, [I, I, I64]),
        "lsa_memindex_score_select": (I, [P, P, P, P, I, P, I64, I, I, I, I, F, P, P, P, P, P, SZ, P]),
        "lsa_memindex_score_select_static": (I, [P, P, P, P, I, P, I64, I, I, I, I, F, P, P, P, P, P]),
        "lsa_fetch_gather": (I, [P, P, P, I64, I, P, SZ, P, P, P, I, I, P, P, P]),
        "lsa_fetch_incremental_workspace_size": (SZ, [I, I64]),
        "lsa_fetch_gather_incremental": (I, [P, P, P, I64, I, P, P, P, I64, P, P, SZ, P, P, P, SZ, P]),
        "lsa_lightning_topk_workspace_size": (SZ, [I, I, I64, I]),
        "lsa_lightning_topk": (I, [P, P, P, P, I, P, P, P, I64, I, I, I, I, I, P, P, P, SZ, P]),
        "lsa_lightning_topk_step_workspace_size": (SZ, [I, I64, I, I, I]),
        "lsa_golden_labels_workspace_size": (SZ, [I, I, I64]),
        "lsa_golden_labels": (I, [P, P, I64, I, I, I, C.c_double, I, P, P, P, SZ, P]),
        "lsa_indexer_train_workspace_size": (SZ, [I, I, I64, I, I, I, I, I]),
        "lsa_indexer_train_step": (I, [P, P, P, P, I, P, P, I, P, P, I64, I, I, I, I, I, I, F, F, P, P, P, P, P, SZ,
                                       P]),
        "lsa_lightning_topk_step": (I, [P, I64, P, I64, P, P, I, P, P, P, I64, P, P, P, I, I, I, I, I, P, P, P, SZ, P]),
        "lsa_pool_alloc": (I, [SZ, C.POINTER(C.c_void_p)]),
        "lsa_pool_free": (I, [P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


_lib = _load()


def library():
    return _lib


def _check(status: int):
    if status != 0:
        raise LSAError(status, _lib.lsa_last_error().decode())


def _p(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the LSA library must be contiguous")
    return t.data_ptr()


def _p_rows(t):
    """Pointer of a view whose rows are contiguous but whose outer (batch) stride may be larger."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    return t.data_ptr()


def _need(dtype, **named):
    """Element types the C ABI reads or writes (include/lsa.h): checked here, since a pointer does
    not carry one and a wrong width would send a kernel past the end of a buffer."""
    for name, t in named.items():
        if t is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _cap(n, **named):
    """Buffers the kernels index up to n elements (sizes from include/lsa.h): too small a buffer
    would be read or written past its end."""
    for name, t in named.items():
        if t is not None and t.numel() < n:
            raise ValueError(f"{name} holds {t.numel()} elements, the call needs {n}")


def _cap_bytes(nbytes, **named):
    for name, t in named.items():
        if t is not None and t.numel() * t.element_size() < nbytes:
            raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, the call needs {nbytes}")


def _offsets(seq_offsets, B):
    _need(torch.int64, seq_offsets=seq_offsets)
    if seq_offsets.numel() != B + 1:
        raise ValueError(f"seq_offsets must hold B + 1 = {B + 1} prefix offsets, got {seq_offsets.numel()}")


def _dev(*ts):
    for t in ts:
        if t is not None and t.device.type != "cuda":
            raise ValueError("device tensor expected (got a CPU tensor)")


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def version() -> str:
    return _lib.lsa_version().decode()


def launch_count() -> int:
    return int(_lib.lsa_launch_count())


def lsa_check_device(stream=None):
    _check(_lib.lsa_check_device(_stream(stream)))


def lsa_selftest_wait_timeout(status_out, stream=None):
    """A bounded wait that nothing completes gives up after 2 s and flags the device error word
    (see include/lsa.h); status_out: device int32 [2]."""
    _need(torch.int32, status_out=status_out)
    _cap(2, status_out=status_out)
    _dev(status_out)
    _check(_lib.lsa_selftest_wait_timeout(_p(status_out), _stream(stream)))


# ------------------------------------------------------------------------ stage 1

def lsa_project_workspace_size(L, B, d, r, n_h, d_I, dt) -> int:
    return int(_lib.lsa_project_workspace_size(L, B, d, r, n_h, d_I, DTYPE_CODE[dt]))


def lsa_project(h, W_dq, W_iuq, W_w, q_out, w_out, workspace, stream=None):
    """c^Q = h W^DQ, q = c^Q W^IUQ, w = h W^w for every layer and sequence (see include/lsa.h)."""
    _need(h.dtype, W_dq=W_dq, W_iuq=W_iuq, W_w=W_w, q_out=q_out)
    _need(torch.float32, w_out=w_out)
    L, B, d = h.shape
    r = W_dq.shape[1]
    _, _, n_h, d_I = q_out.shape
    _dev(h, W_dq, W_iuq, W_w, q_out, w_out, workspace)
    _check(_lib.lsa_project(_p(h), _p(W_dq), _p(W_iuq), _p(W_w), DTYPE_CODE[h.dtype], L, B, d, r, n_h, d_I,
                            _p(q_out), _p(w_out), _p(workspace), workspace.numel() * workspace.element_size(),
                            _stream(stream)))


# ------------------------------------------------------------------------ stages 2-4a

def lsa_score_select_workspace_size(L, B, total_S) -> int:
    return int(_lib.lsa_score_select_workspace_size(L, B, total_S))


def _score_select_types(q, w, K, k_scale, seq_offsets, total_S, idx_out, count_out, scores_out, mask_out):
    _need(torch.float32 if K.dtype == torch.float32 else torch.bfloat16, q=q)
    _need(torch.float32, w=w, k_scale=k_scale, scores_out=scores_out)
    _need(torch.int32, idx_out=idx_out, count_out=count_out)
    _need(torch.uint8, mask_out=mask_out)
    _offsets(seq_offsets, q.shape[1])
    L, B, n_h, d_I = q.shape
    T = int(total_S)
    if K.shape[1] < T:
        raise ValueError(f"K holds {K.shape[1]} entries per layer, total_S is {T}")
    _cap(L * B * n_h, w=w)
    _cap(L * T, k_scale=k_scale, scores_out=scores_out)
    _cap(T, idx_out=idx_out, mask_out=mask_out)
    _cap(B, count_out=count_out)


def lsa_memindex_score_select(q, w, K, k_scale, seq_offsets, total_S, threshold, idx_out, count_out,
                              workspace, scores_out=None, mask_out=None, stream=None):
    """Index score, threshold, OR over layers and compaction (see include/lsa.h)."""
    _score_select_types(q, w, K, k_scale, seq_offsets, total_S, idx_out, count_out, scores_out, mask_out)
    L, B, n_h, d_I = q.shape
    _dev(q, w, K, k_scale, seq_offsets, idx_out, count_out, workspace, scores_out, mask_out)
    _check(_lib.lsa_memindex_score_select(
        _p(q), _p(w), _p(K), _p(k_scale), DTYPE_CODE[K.dtype], _p(seq_offsets), int(total_S), L, B, n_h, d_I,
        float(threshold), _p(scores_out), _p(mask_out), _p(idx_out), _p(count_out), _p(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


STATIC_SCORE_SCRATCH_BYTES = 8 << 20  # LSA_STATIC_SCORE_SCRATCH_BYTES in include/lsa.h


def lsa_memindex_score_select_static(q, w, K, k_scale, seq_offsets, total_S, threshold, idx_out, count_out,
                                     scores_out=None, mask_out=None, stream=None):
    """lsa_memindex_score_select with the library's own per-device scratch instead of a workspace:
    the call allocates nothing (see include/lsa.h for the size limit and the ordering rule)."""
    _score_select_types(q, w, K, k_scale, seq_offsets, total_S, idx_out, count_out, scores_out, mask_out)
    L, B, n_h, d_I = q.shape
    _dev(q, w, K, k_scale, seq_offsets, idx_out, count_out, scores_out, mask_out)
    _check(_lib.lsa_memindex_score_select_static(
        _p(q), _p(w), _p(K), _p(k_scale), DTYPE_CODE[K.dtype], _p(seq_offsets), int(total_S), L, B, n_h, d_I,
        float(threshold), _p(scores_out), _p(mask_out), _p(idx_out), _p(count_out), _stream(stream)))


# ------------------------------------------------------------------------ stage 4b

def lsa_fetch_gather(idx, count, seq_offsets, total_S, pool, hot_kv, K_sel=None, k_scale_sel=None,
                     hot_K=None, hot_scale=None, stream=None):
    """Gather fetched rows from the mapped host cold pool and/or the keys of one layer (pool and
    hot_kv None: keys only; K_sel None: rows only, a small launch meant for a second stream)."""
    _need(torch.int32, idx=idx, count=count)
    _offsets(seq_offsets, count.numel())
    _need(torch.float32, k_scale_sel=k_scale_sel, hot_scale=hot_scale)
    if K_sel is not None:
        _need(torch.bfloat16 if K_sel.dtype == torch.float8_e4m3fn else K_sel.dtype, hot_K=hot_K)
    if pool is not None and pool.device.type != "cpu":
        raise ValueError("the cold pool must be (mapped page-locked) host memory")
    B = count.numel()
    row_bytes = pool.shape[1] * pool.element_size() if pool is not None else 0
    kdt = DTYPE_CODE[K_sel.dtype] if K_sel is not None else 0
    d_I = K_sel.shape[-1] if K_sel is not None else 0
    T = int(total_S)
    _cap(T, idx=idx, k_scale_sel=k_scale_sel, hot_scale=hot_scale)
    _cap(T * d_I, K_sel=K_sel, hot_K=hot_K)
    if pool is not None:
        _cap_bytes(T * row_bytes, pool=pool, hot_kv=hot_kv)
    _dev(idx, count, seq_offsets, hot_kv, K_sel, k_scale_sel, hot_K, hot_scale)
    _check(_lib.lsa_fetch_gather(_p(idx), _p(count), _p(seq_offsets), int(total_S), B, _p(pool), row_bytes,
                                 _p(hot_kv), _p(K_sel), _p(k_scale_sel), kdt, d_I, _p(hot_K), _p(hot_scale),
                                 _stream(stream)))


def lsa_fetch_incremental_workspace_size(B, total_S) -> int:
    return int(_lib.lsa_fetch_incremental_workspace_size(B, total_S))


def lsa_fetch_gather_incremental(idx, count, seq_offsets, total_S, prev_idx, prev_count, prev_seq_offsets,
                                 prev_total_S, prev_hot_kv, pool, hot_kv, workspace, host_rows_out=None,
                                 stream=None):
    """The window's rows with the previous window's rows resident: common entries are copied on the
    device, only the others cross the host link (see include/lsa.h)."""
    _need(torch.int32, idx=idx, count=count, prev_idx=prev_idx, prev_count=prev_count, host_rows_out=host_rows_out)
    _offsets(seq_offsets, count.numel())
    _offsets(prev_seq_offsets, prev_count.numel())
    if pool.device.type != "cpu":
        raise ValueError("the cold pool must be (mapped page-locked) host memory")
    B = count.numel()
    row_bytes = pool.shape[1] * pool.element_size()
    _cap(int(total_S), idx=idx)
    _cap(int(prev_total_S), prev_idx=prev_idx)
    _cap(1, host_rows_out=host_rows_out)
    _cap_bytes(int(total_S) * row_bytes, pool=pool, hot_kv=hot_kv)
    _cap_bytes(int(prev_total_S) * row_bytes, prev_hot_kv=prev_hot_kv)
    _dev(idx, count, seq_offsets, prev_idx, prev_count, prev_seq_offsets, prev_hot_kv, hot_kv, workspace,
         host_rows_out)
    _check(_lib.lsa_fetch_gather_incremental(
        _p(idx), _p(count), _p(seq_offsets), int(total_S), B, _p(prev_idx), _p(prev_count), _p(prev_seq_offsets),
        int(prev_total_S), _p(prev_hot_kv), _p(pool), row_bytes, _p(hot_kv), _p(host_rows_out), _p(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


# ------------------------------------------------------------------------ stage 5

def lsa_lightning_topk_workspace_size(B, tau, total_S, k) -> int:
    return int(_lib.lsa_lightning_topk_workspace_size(B, tau, total_S, k))


def lsa_lightning_topk(q_dec, w_dec, hot_K, hot_scale, idx, count, seq_offsets, total_S, k, topk_idx,
                       workspace, topk_score=None, stream=None):
    """Native Lightning-Indexer Top-k over the fetched entries (see include/lsa.h).  With E4M3
    keys, hot_K is the bf16 decode written by lsa_fetch_gather and hot_scale holds the scales."""
    _need(torch.float32 if hot_K.dtype == torch.float32 else torch.bfloat16, q_dec=q_dec)
    _need(torch.float32, w_dec=w_dec, hot_scale=hot_scale, topk_score=topk_score)
    _need(torch.int32, idx=idx, count=count, topk_idx=topk_idx)
    _offsets(seq_offsets, q_dec.shape[0])
    B, tau, n_h, d_I = q_dec.shape
    kdt = LSA_FP8_E4M3 if hot_scale is not None else DTYPE_CODE[hot_K.dtype]
    T = int(total_S)
    _cap(B * tau * n_h, w_dec=w_dec)
    _cap(T, idx=idx, hot_scale=hot_scale)
    _cap(T * d_I, hot_K=hot_K)
    _cap(B, count=count)
    _cap(B * tau * int(k), topk_idx=topk_idx, topk_score=topk_score)
    _dev(q_dec, w_dec, hot_K, hot_scale, idx, count, seq_offsets, topk_idx, workspace, topk_score)
    _check(_lib.lsa_lightning_topk(_p(q_dec), _p(w_dec), _p(hot_K), _p(hot_scale), kdt,
                                   _p(idx), _p(count), _p(seq_offsets), int(total_S), B, tau, n_h, d_I, int(k),
                                   _p(topk_idx), _p(topk_score), _p(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))


# ------------------------------------------------------------------------ golden labels, training step

def lsa_golden_labels_workspace_size(tau, Lc, total_S) -> int:
    return int(_lib.lsa_golden_labels_workspace_size(tau, Lc, total_S))


def lsa_golden_labels(z, seq_offsets, label_out, workspace, p=0.6, theta=3, nsize_out=None, stream=None):
    """Golden labels of one window from raw indexer logits z [tau][Lc][T] fp32 (see include/lsa.h)."""
    _need(torch.float32, z=z)
    _need(torch.uint8, label_out=label_out)
    _need(torch.int32, nsize_out=nsize_out)
    _need(torch.int64, seq_offsets=seq_offsets)
    tau, Lc, T = z.shape
    B = seq_offsets.numel() - 1
    _cap(T, label_out=label_out)
    _cap(B * tau * Lc, nsize_out=nsize_out)
    _dev(z, seq_offsets, label_out, workspace, nsize_out)
    _check(_lib.lsa_golden_labels(_p(z), _p(seq_offsets), T, B, tau, Lc, float(p), int(theta), _p(label_out),
                                  _p(nsize_out), _p(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream)))


def lsa_indexer_train_workspace_size(L, B, total_S, d, r, n_h, d_I, dtype) -> int:
    return int(_lib.lsa_indexer_train_workspace_size(L, B, total_S, d, r, n_h, d_I, DTYPE_CODE[dtype]))


def lsa_indexer_train_step(h, W_dq, W_iuq, W_w, K, k_scale, labels, seq_offsets, loss_out, g_Wdq, g_Wiuq, g_Ww,
                           workspace, n_h, d_I, gamma=0.0, alpha=-1.0, stream=None):
    """Loss and gradients of W^DQ, W^IUQ, W^w for one training step (see include/lsa.h)."""
    _need(h.dtype, W_dq=W_dq, W_iuq=W_iuq, W_w=W_w)
    _need(torch.float32, k_scale=k_scale, g_Wdq=g_Wdq, g_Wiuq=g_Wiuq, g_Ww=g_Ww)
    _need(torch.uint8, labels=labels)
    _need(torch.float64, loss_out=loss_out)
    _offsets(seq_offsets, h.shape[1])
    L, B, d = h.shape
    r = W_dq.shape[1]
    T = K.shape[1]
    _cap(T, labels=labels)
    _cap(L * T, k_scale=k_scale)
    _cap(1, loss_out=loss_out)
    _cap(W_dq.numel(), g_Wdq=g_Wdq)
    _cap(W_iuq.numel(), g_Wiuq=g_Wiuq)
    _cap(W_w.numel(), g_Ww=g_Ww)
    _dev(h, W_dq, W_iuq, W_w, K, k_scale, labels, seq_offsets, loss_out, g_Wdq, g_Wiuq, g_Ww, workspace)
    _check(_lib.lsa_indexer_train_step(
        _p(h), _p(W_dq), _p(W_iuq), _p(W_w), DTYPE_CODE[h.dtype], _p(K), _p(k_scale), DTYPE_CODE[K.dtype], _p(labels),
        _p(seq_offsets), T, L, B, d, r, n_h, d_I, float(gamma), float(alpha), _p(loss_out), _p(g_Wdq), _p(g_Wiuq),
        _p(g_Ww), _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def lsa_lightning_topk_step_workspace_size(B, total_S, n_h, d_I, W) -> int:
    return int(_lib.lsa_lightning_topk_step_workspace_size(B, total_S, n_h, d_I, W))


def lsa_lightning_topk_step(q_step, w_step, hot_K, hot_scale, idx, count, seq_offsets, total_S, k, topk_idx,
                            workspace, win_K=None, win_scale=None, win_count=None, topk_score=None, kdt=None,
                            stream=None):
    """One decode step: q_step [B][n_h][d_I] and w_step [B][n_h] may be strided views (e.g. a
    column q_dec[:, i] of the window's queries); window entries win_K [B][W][d_I] with win_count [B]."""
    _need(torch.float32 if hot_K.dtype == torch.float32 else torch.bfloat16, q_step=q_step)
    _need(hot_K.dtype, win_K=win_K)
    _need(torch.float32, w_step=w_step, hot_scale=hot_scale, win_scale=win_scale, topk_score=topk_score)
    _need(torch.int32, idx=idx, count=count, win_count=win_count, topk_idx=topk_idx)
    _offsets(seq_offsets, q_step.shape[0])
    B, n_h, d_I = q_step.shape
    if q_step.stride(2) != 1 or q_step.stride(1) != d_I or w_step.stride(1) != 1:
        raise ValueError("q_step rows and w_step rows must be contiguous (a batch stride is allowed)")
    if kdt is None:
        kdt = DTYPE_CODE[torch.float8_e4m3fn] if hot_scale is not None else DTYPE_CODE[hot_K.dtype]
    W = win_K.shape[1] if win_K is not None else 0
    T = int(total_S)
    _cap(T, idx=idx, hot_scale=hot_scale)
    _cap(T * d_I, hot_K=hot_K)
    _cap(B, count=count, win_count=win_count)
    _cap(B * W, win_scale=win_scale)
    _cap(B * int(k), topk_idx=topk_idx, topk_score=topk_score)
    _dev(q_step, w_step, hot_K, hot_scale, idx, count, seq_offsets, topk_idx, workspace, win_K, win_scale, win_count,
         topk_score)
    _check(_lib.lsa_lightning_topk_step(
        _p_rows(q_step), q_step.stride(0), _p_rows(w_step), w_step.stride(0), _p(hot_K), _p(hot_scale), kdt, _p(idx), _p(count),
        _p(seq_offsets), int(total_S), _p(win_K), _p(win_scale), _p(win_count), W, B, n_h, d_I, int(k), _p(topk_idx),
        _p(topk_score), _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


# ------------------------------------------------------------------------ cold pool

class MappedPool:
    """Mapped page-locked host buffer from lsa_pool_alloc, viewed as a uint8 tensor [rows][row_bytes]."""

    def __init__(self, rows: int, row_bytes: int):
        ptr = C.c_void_p()
        _check(_lib.lsa_pool_alloc(rows * row_bytes, C.byref(ptr)))
        self.ptr = ptr.value
        self.nbytes = rows * row_bytes
        arr = (C.c_uint8 * self.nbytes).from_address(self.ptr)
        self.tensor = torch.frombuffer(arr, dtype=torch.uint8).view(rows, row_bytes)

    def free(self):
        if self.ptr:
            self.tensor = None
            _check(_lib.lsa_pool_free(self.ptr))
            self.ptr = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass

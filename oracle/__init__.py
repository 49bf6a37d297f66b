"""CPU oracle of the Lookahead Sparse Attention indexer path -- TEST INFRASTRUCTURE.

Thin ctypes wrapper over ``oracle/lsa_oracle.c`` (plain scalar C, double precision), which
restates the method from the source pages step by step; see that file's header for the
passages each function follows.  Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library neither imports
nor links it, and this package imports nothing from the library.
"""
from __future__ import annotations

import ctypes as C
import numpy as np
import torch

from . import build as _build

DT = {"f32": 0, "bf16": 1, "fp8": 2, "f64": 3}   # f64: exact inputs, for the training-step pins only
_TORCH_DT = {torch.float32: "f32", torch.bfloat16: "bf16", torch.float8_e4m3fn: "fp8", torch.float64: "f64"}

_lib = None


def _load(path):
    h = C.CDLL(path)
    P, I, I64, D = C.c_void_p, C.c_int, C.c_int64, C.c_double
    h.lsa_oracle_bf16_bits.restype = C.c_uint16
    h.lsa_oracle_bf16_bits.argtypes = [D]
    h.lsa_oracle_bf16_round_array.argtypes = [P, P, I64]
    h.lsa_oracle_e4m3_decode_array.argtypes = [P, P, I64]
    h.lsa_oracle_sigmoid.restype = D
    h.lsa_oracle_sigmoid.argtypes = [D]
    h.lsa_oracle_threads.restype = I
    h.lsa_oracle_set_threads.argtypes = [I]
    h.lsa_oracle_project.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, P, P]
    h.lsa_oracle_score.argtypes = [P, I, P, P, P, I, P, I, I, I, I, D, P, P, P, P, P]
    h.lsa_oracle_score_entries.argtypes = [P, I, P, P, P, I, P, I, I, I, I, I64, P, P, P]
    h.lsa_oracle_gather.argtypes = [P, P, P, I, P, I64, P, P, P, I, I, P, P]
    h.lsa_oracle_lightning_topk.argtypes = [P, I, P, P, P, I, P, P, P, I, I, I, I, I, I64, P, P, P, P, P]
    h.lsa_oracle_golden_labels.argtypes = [P, P, I, I, I, D, I, P, P, P]
    h.lsa_oracle_train_step.argtypes = [P, P, P, P, I, P, P, I, P, P, I, I, I, I, I, I, D, D, P, P, P, P]
    for f in ("project", "score", "score_entries", "gather", "lightning_topk"):
        getattr(h, "lsa_oracle_" + f).restype = I
    h.lsa_oracle_golden_labels.restype = I
    h.lsa_oracle_train_step.restype = I
    return h


class using:
    """Context manager: run the wrapper against another build of the oracle source (the
    test suite uses it to check that deliberately broken copies fail the pins)."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = _load(self.path)
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def lib():
    global _lib
    if _lib is None:
        _lib = _load(_build.build())
    return _lib


def threads() -> int:
    return lib().lsa_oracle_threads()


def set_threads(n: int) -> None:
    lib().lsa_oracle_set_threads(int(n))


def _c(t):
    """Contiguous CPU buffer (torch tensor or numpy array) -> (keepalive, address)."""
    if t is None:
        return None, None
    if isinstance(t, torch.Tensor):
        t = t.detach().contiguous()
        if t.device.type != "cpu":
            raise ValueError("oracle inputs must be CPU tensors")
        return t, t.data_ptr()
    a = np.ascontiguousarray(t)
    return a, a.ctypes.data


def _dt(t) -> int:
    return DT[_TORCH_DT[t.dtype]]


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


# ---------------------------------------------------------------- storage helpers

def bf16_bits(x) -> np.ndarray:
    """Nearest-even bf16 of real values (float64 array) as uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().lsa_oracle_bf16_round_array(x.ctypes.data, out.ctypes.data, x.size)
    return out


def e4m3_decode(codes) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    lib().lsa_oracle_e4m3_decode_array(codes.ctypes.data, out.ctypes.data, codes.size)
    return out


def sigmoid(x: float) -> float:
    return lib().lsa_oracle_sigmoid(float(x))


# ---------------------------------------------------------------- the path, stage by stage

def project(h, W_dq, W_iuq, W_w, n_h: int, d_I: int, want_c: bool = False):
    """c = h W^DQ, q = c W^IUQ (both stored in h's dtype), w = h W^w (fp32).

    h [L][B][d]; W_dq [L][r][d]; W_iuq [L][n_h*d_I][r]; W_w [L][n_h][d] (rows = outputs).
    Returns q [L][B][n_h][d_I] (torch, h's dtype), w [L][B][n_h] float32 (, c [L][B][r]).
    """
    L, B, d = h.shape
    r = W_dq.shape[1]
    q = torch.empty((L, B, n_h, d_I), dtype=h.dtype)
    w = torch.empty((L, B, n_h), dtype=torch.float32)
    c = torch.empty((L, B, r), dtype=h.dtype) if want_c else None
    ks = [_c(x) for x in (h, W_dq, W_iuq, W_w)]
    rc = lib().lsa_oracle_project(ks[0][1], ks[1][1], ks[2][1], ks[3][1], _dt(h), L, B, d, r, n_h, d_I,
                                  q.data_ptr(), w.data_ptr(), c.data_ptr() if c is not None else None)
    _check(rc, "project")
    return (q, w, c) if want_c else (q, w)


def score(q, w, K, k_scale, seq_offsets, threshold: float = 0.5, want_x: bool = True):
    """Fetch decision for every entry ([L] layers OR-combined) and the fetched list.

    Returns dict: x [L][T] logits, I [L][T] sigmoid scores, mask [T] uint8, idx [T] int32
    (ascending s per sequence, first count[b] slots of segment b, rest -1), count [B].
    """
    L, B, n_h, d_I = q.shape
    offs = np.ascontiguousarray(seq_offsets, dtype=np.int64)
    T = int(offs[-1])
    x = np.empty((L, T), dtype=np.float64) if want_x else None
    I = np.empty((L, T), dtype=np.float64) if want_x else None
    mask = np.empty(T, dtype=np.uint8)
    idx = np.full(T, -1, dtype=np.int32)
    cnt = np.empty(B, dtype=np.int32)
    kq, kw, kK, ks, ko = _c(q), _c(w), _c(K), _c(k_scale), _c(offs)
    rc = lib().lsa_oracle_score(kq[1], _dt(q), kw[1], kK[1], ks[1], _dt(K), ko[1], L, B, n_h, d_I,
                                float(threshold), x.ctypes.data if x is not None else None,
                                I.ctypes.data if I is not None else None, mask.ctypes.data,
                                idx.ctypes.data, cnt.ctypes.data)
    _check(rc, "score")
    return {"x": x, "I": I, "mask": mask, "idx": idx, "count": cnt}


def score_entries(q, w, K, k_scale, seq_offsets, ent_b, ent_s) -> np.ndarray:
    """Logits x [L][n] of sampled entries (ent_b[i], ent_s[i])."""
    L, B, n_h, d_I = q.shape
    offs = np.ascontiguousarray(seq_offsets, dtype=np.int64)
    eb = np.ascontiguousarray(ent_b, dtype=np.int32)
    es = np.ascontiguousarray(ent_s, dtype=np.int64)
    out = np.empty((L, eb.size), dtype=np.float64)
    kq, kw, kK, ks, ko = _c(q), _c(w), _c(K), _c(k_scale), _c(offs)
    rc = lib().lsa_oracle_score_entries(kq[1], _dt(q), kw[1], kK[1], ks[1], _dt(K), ko[1], L, B, n_h, d_I,
                                        eb.size, eb.ctypes.data, es.ctypes.data, out.ctypes.data)
    _check(rc, "score_entries")
    return out


def gather(idx, count, seq_offsets, pool=None, K_sel=None, k_scale_sel=None, d_I: int = 0):
    """Byte copies of the fetched rows (pool rows, keys and scales of the selected layer).

    Returns (hot_kv [T][row_bytes] uint8 or None, hot_K [T][d_I] or None, hot_scale or None);
    slots past count[b] are zero.
    """
    offs = np.ascontiguousarray(seq_offsets, dtype=np.int64)
    T = int(offs[-1])
    B = offs.size - 1
    hot_kv = torch.zeros((T, pool.shape[1]), dtype=torch.uint8) if pool is not None else None
    hot_K = torch.zeros((T, K_sel.shape[1]), dtype=K_sel.dtype) if K_sel is not None else None
    hot_sc = torch.zeros(T, dtype=torch.float32) if k_scale_sel is not None else None
    ki, kc, ko, kp, kK, ks = _c(idx), _c(count), _c(offs), _c(pool), _c(K_sel), _c(k_scale_sel)
    rc = lib().lsa_oracle_gather(ki[1], kc[1], ko[1], B, kp[1], pool.shape[1] if pool is not None else 0,
                                 hot_kv.data_ptr() if hot_kv is not None else None, kK[1], ks[1],
                                 _dt(K_sel) if K_sel is not None else 0,
                                 K_sel.shape[1] if K_sel is not None else 0,
                                 hot_K.data_ptr() if hot_K is not None else None,
                                 hot_sc.data_ptr() if hot_sc is not None else None)
    _check(rc, "gather")
    return hot_kv, hot_K, hot_sc


def lightning_topk(q_dec, w_dec, K_sel, k_scale_sel, idx, count, seq_offsets, k: int,
                   queries=None, want_y: bool = False):
    """Native Lightning-Indexer Top-k over the fetched entries of each sequence.

    q_dec [B][tau][n_h][d_I]; w_dec [B][tau][n_h]; K_sel [T][d_I] keys of the selected layer.
    queries: optional list of (b, i) pairs (default: all B*tau queries, b-major).
    Returns dict: idx [n][k] int32 (entry s, -1 pad), score [n][k] float64 (-inf pad),
    y [n][T] (when want_y: scores of sequence b at columns seq_offsets[b] + j).
    """
    B, tau, n_h, d_I = q_dec.shape
    offs = np.ascontiguousarray(seq_offsets, dtype=np.int64)
    T = int(offs[-1])
    if queries is None:
        nq, qb, qi = -1, None, None
        n = B * tau
    else:
        qa = np.asarray(queries, dtype=np.int32).reshape(-1, 2)
        qb, qi = np.ascontiguousarray(qa[:, 0]), np.ascontiguousarray(qa[:, 1])
        nq = n = qa.shape[0]
    out_i = np.empty((n, k), dtype=np.int32)
    out_s = np.empty((n, k), dtype=np.float64)
    y = np.zeros((n, T), dtype=np.float64) if want_y else None
    kq, kw, kK, ks, ki, kc, ko = (_c(q_dec), _c(w_dec), _c(K_sel), _c(k_scale_sel), _c(idx), _c(count), _c(offs))
    rc = lib().lsa_oracle_lightning_topk(kq[1], _dt(q_dec), kw[1], kK[1], ks[1], _dt(K_sel), ki[1], kc[1], ko[1],
                                         B, tau, n_h, d_I, int(k), nq,
                                         qb.ctypes.data if qb is not None else None,
                                         qi.ctypes.data if qi is not None else None,
                                         out_i.ctypes.data, out_s.ctypes.data,
                                         y.ctypes.data if y is not None else None)
    _check(rc, "lightning_topk")
    return {"idx": out_i, "score": out_s, "y": y}


def golden_labels(z, seq_offsets, p: float = 0.6, theta: int = 3, want_golden: bool = False):
    """Golden labels of one future window from raw indexer logits z [tau][Lc][T] (float32).

    Returns dict: label [T] uint8 (golden for some token of the window), nsize [B][tau][Lc] int32
    (nucleus sizes), golden [tau][T] uint8 when want_golden.
    """
    tau, Lc, T = z.shape
    offs = np.ascontiguousarray(seq_offsets, dtype=np.int64)
    B = offs.size - 1
    zz = np.ascontiguousarray(z.numpy() if hasattr(z, "numpy") else z, dtype=np.float32)
    label = np.zeros(T, dtype=np.uint8)
    nsize = np.zeros((B, tau, Lc), dtype=np.int32)
    golden = np.zeros((tau, T), dtype=np.uint8) if want_golden else None
    rc = lib().lsa_oracle_golden_labels(zz.ctypes.data, offs.ctypes.data, B, tau, Lc, float(p), int(theta),
                                        label.ctypes.data, golden.ctypes.data if golden is not None else None,
                                        nsize.ctypes.data)
    _check(rc, "golden_labels")
    return {"label": label, "nsize": nsize, "golden": golden}


def train_step(h, W_dq, W_iuq, W_w, K, k_scale, labels, seq_offsets, n_h: int, d_I: int, gamma: float = 0.0,
               alpha: float = -1.0):
    """Loss and gradients of one indexer training step (focal loss; gamma = 0, alpha < 0 is BCE).

    h [L][B][d], W_dq [L][r][d], W_iuq [L][n_h*d_I][r], W_w [L][n_h][d] (one dtype: f32, bf16 or
    f64 = exact); K [L][T][d_I], k_scale [L][T] or None; labels [T] (0/1).
    Returns dict: loss (float), g_Wdq, g_Wiuq, g_Ww (float64 arrays in the weights' shapes).
    """
    L, B, d = h.shape
    r = W_dq.shape[1]
    offs = np.ascontiguousarray(seq_offsets, dtype=np.int64)
    lab = np.ascontiguousarray(np.asarray(labels), dtype=np.uint8)
    g_dq = np.zeros(tuple(W_dq.shape), dtype=np.float64)
    g_iuq = np.zeros(tuple(W_iuq.shape), dtype=np.float64)
    g_w = np.zeros(tuple(W_w.shape), dtype=np.float64)
    loss = np.zeros(1, dtype=np.float64)
    ks = [_c(x) for x in (h, W_dq, W_iuq, W_w, K, k_scale)]
    rc = lib().lsa_oracle_train_step(ks[0][1], ks[1][1], ks[2][1], ks[3][1], _dt(h), ks[4][1], ks[5][1], _dt(K),
                                     lab.ctypes.data, offs.ctypes.data, L, B, d, r, n_h, d_I, float(gamma),
                                     float(alpha), loss.ctypes.data, g_dq.ctypes.data, g_iuq.ctypes.data,
                                     g_w.ctypes.data)
    _check(rc, "train_step")
    return {"loss": float(loss[0]), "g_Wdq": g_dq, "g_Wiuq": g_iuq, "g_Ww": g_w}

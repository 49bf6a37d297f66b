"""Seeded synthetic inputs for the Lookahead Sparse Attention indexer path.

This module only *draws* inputs: hidden states, indexer projection weights, compressed
index keys K^IComp (with their FP8 encoding and per-entry scales), the CPU cold-pool KV
rows, and the decode-step queries of the native Lightning Indexer.  It computes none of
the indexer's outputs (no projection of data, no index score, no threshold, no Top-k), so
both the CUDA path and the CPU oracle can consume the same inputs without sharing any of
the method's arithmetic.

Workload shapes follow the page "FlashMemory-DeepSeek-V4: 13.5% of the memory ..." (blog
review), section 3 (trigger every tau = 64 decode steps, three indexer layers 10/12/20,
low-rank query projection) and the hyper.ai summary's dataset paragraph (contexts of
16K-512K tokens).  Fetch rates are steered toward the 13.5 % average footprint of that
review's section 5 table, or a per-sequence rate from 1 % to 40 % for the ragged mix.

Planted entries (workloads with ``planted > 0``): each layer has one unit direction u_h per
head, drawn by the generator.  The projection weights carry it: column 0 of W^IUQ holds
(sqrt(d_I) / PLANT_ALPHA) u_h in head h's rows, and every hidden state is built so that
c^Q[0] = h W^DQ[0] equals PLANT_ALPHA (the same linear construction that pins h W^w to the drawn
head weights), so the queries that stage 1 produces contain sqrt(d_I) u_h; the stage-level query
draws contain the same component.  A planted key of sequence b is cos * v + sqrt(1 - cos^2) * n,
v = normalise(sum_h w_h u_h) with the sequence's own head weights w and n a unit vector
orthogonal to v: it lifts the heads of positive weight and sinks those of negative weight.
None of this evaluates a projection or a score.

Fetch-rate calibration: the head-weight shift comes from a normal model of the score of random
keys; the fetch rate it gives through the whole path (stage 1 included) differs from the target
by a few percent of the entries.  ``fetch_calibration.json`` holds, per workload, seed and
sequence, the model target that gives the wanted rate through the whole path on that
sequence's own inputs (written by ``tests/calibrate_fetch.py`` with the CPU oracle); it is used
when the workload's name, seed and target match, and the target is used as is otherwise.

Determinism: every tensor slice is drawn from its own ``numpy.random.default_rng`` stream
keyed by (seed, part, layer, sequence), so a subset of sequences can be regenerated alone
and is bit-identical to the same sequences of the full batch.
"""
from __future__ import annotations

import json
import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "workload", "Inputs", "make_inputs", "DTYPES"]

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.float8_e4m3fn}
# numeric codes shared by the C ABI of the library and of the oracle (LSA_F32, LSA_BF16,
# LSA_FP8_E4M3); this is an interface constant, not arithmetic.
DTYPE_CODE = {"f32": 0, "bf16": 1, "fp8": 2}

_PART = {"h": 1, "wdq": 2, "wiuq": 3, "ww": 4, "key": 5, "plant": 6, "pool": 7,
         "q": 8, "w": 9, "qdec": 10, "wdec": 11, "lens": 12, "rate": 13, "pdir": 14}

# Planted direction in the queries: c^Q[0] = PLANT_ALPHA and W^IUQ[:, 0] = (sqrt(d_I) / PLANT_ALPHA) u_h,
# so the planted component of every head's query is sqrt(d_I) u_h, as long as the random part of a
# query with unit-variance elements.
PLANT_ALPHA = 4.0

_THREADS = 8


@dataclass(frozen=True)
class Workload:
    """Shape and distribution recipe of one synthetic workload."""
    name: str
    B: int                      # sequences (independent trigger steps)
    L: int                      # memory-indexer layers (OR-combined)
    S: tuple                    # compressed entries per sequence, per layer
    d: int                      # hidden size
    r: int                      # query down-projection rank
    n_h: int                    # indexer heads
    d_I: int                    # indexer head dim
    tau: int                    # decode queries per trigger window
    k: int                      # Lightning-Indexer Top-k
    row_bytes: int              # bytes of one compressed KV row in the cold pool
    dtype: str                  # h, weights and queries: "f32" or "bf16"
    kdtype: str                 # K^IComp: "f32", "bf16" or "fp8"
    fetch: tuple                # per-sequence target fetch fraction (after the OR)
    planted: float = 0.0        # fraction of entries planted along the queries' planted directions
    planted_run: tuple = (1, 1) # planted entries come in runs of this length range
    planted_cos: float = 0.6
    seed: int = 1000
    sel_layer: int = 0          # layer whose keys the decode-step Lightning Indexer uses

    @property
    def total_S(self) -> int:
        return int(sum(self.S))

    @property
    def seq_offsets(self) -> np.ndarray:
        o = np.zeros(self.B + 1, dtype=np.int64)
        o[1:] = np.cumsum(np.asarray(self.S, dtype=np.int64))
        return o

    def subset(self, seqs) -> "Workload":
        """The same workload restricted to some sequences (values are unchanged)."""
        seqs = list(seqs)
        return replace(self, B=len(seqs), S=tuple(self.S[b] for b in seqs),
                       fetch=tuple(self.fetch[b] for b in seqs),
                       name=f"{self.name}[{','.join(map(str, seqs))}]",
                       _seq_ids=tuple(self._ids()[b] for b in seqs))

    # original sequence ids (so subsets keep their random streams)
    _seq_ids: tuple = field(default=(), compare=False)

    def _ids(self):
        return self._seq_ids if self._seq_ids else tuple(range(self.B))


def _ragged_lengths(seed: int, B: int):
    rng = np.random.default_rng([seed, _PART["lens"]])
    ctx = np.exp(rng.uniform(math.log(16 * 1024), math.log(512 * 1024), size=B))
    S = np.clip(np.floor(ctx / 4).astype(np.int64), 4096, 131072)
    rates = np.random.default_rng([seed, _PART["rate"]]).uniform(0.01, 0.40, size=B)
    return tuple(int(s) for s in S), tuple(float(x) for x in rates)


def _build_workloads():
    big = dict(d=4096, r=2048, n_h=64, d_I=128, row_bytes=1024, dtype="bf16")
    w = {}
    w["tiny_fp32"] = Workload("tiny_fp32", B=1, L=1, S=(512,), d=256, r=64, n_h=4, d_I=32,
                              tau=4, k=16, row_bytes=256, dtype="f32", kdtype="f32",
                              fetch=(0.15,), seed=1000)
    w["ctx128k_bf16"] = Workload("ctx128k_bf16", B=1, L=3, S=(32768,), tau=64, k=512,
                                 kdtype="bf16", fetch=(0.135,), planted=0.02, seed=1001, **big)
    w["ctx500k_bf16_b8"] = Workload("ctx500k_bf16_b8", B=8, L=3, S=(131072,) * 8, tau=64,
                                    k=1024, kdtype="bf16", fetch=(0.135,) * 8, seed=1002, **big)
    w["ctx1m_fp8_b32"] = Workload("ctx1m_fp8_b32", B=32, L=3, S=(262144,) * 32, tau=64,
                                  k=2048, kdtype="fp8", fetch=(0.135,) * 32, planted=0.02,
                                  planted_run=(8, 64), seed=1003, **big)
    S5, rates5 = _ragged_lengths(1004, 64)
    w["ragged_mix_b64"] = Workload("ragged_mix_b64", B=64, L=3, S=S5, tau=64, k=512,
                                   kdtype="bf16", fetch=rates5, seed=1004, **big)
    return w


WORKLOADS = _build_workloads()


def workload(base: str, **overrides) -> Workload:
    """A named workload, optionally with fields replaced (B alone repeats the base lengths)."""
    wl = WORKLOADS[base]
    if "B" in overrides and "S" not in overrides:
        B = overrides["B"]
        overrides["S"] = tuple(wl.S[i % wl.B] for i in range(B))
        overrides["fetch"] = tuple(wl.fetch[i % wl.B] for i in range(B))
    return replace(wl, **overrides) if overrides else wl


# --------------------------------------------------------------------------- helpers

def _rng(wl: Workload, part: str, *key):
    return np.random.default_rng([wl.seed, _PART[part], *key])


_POOL = ThreadPoolExecutor(_THREADS)
_CHUNK_ELEMS = 1 << 20


def _normal_rows(wl: Workload, part: str, key: tuple, rows: int, cols: int, scale: float = 1.0,
                 out: np.ndarray = None) -> np.ndarray:
    """rows x cols float32 N(0, scale^2); each block of about 2^20 elements (whole rows) has
    its own stream (seed, part, *key, block), so the result does not depend on threading."""
    if out is None:
        out = np.empty((rows, cols), dtype=np.float32)
    step = max(1, _CHUNK_ELEMS // cols)

    def fill(c0):
        blk = out[c0:c0 + step]
        _rng(wl, part, *key, c0 // step).standard_normal(blk.shape, dtype=np.float32, out=blk)
        if scale != 1.0:
            blk *= np.float32(scale)

    list(_POOL.map(fill, range(0, rows, step)))
    return out


def _cast(x: np.ndarray, dt: str) -> torch.Tensor:
    """float32/float64 numpy -> torch tensor of the storage dtype (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(DTYPES[dt])


def _phi(z: float) -> float:
    return 0.5 * math.erfc(-z / math.sqrt(2.0))


def _shift_for_rate(g: np.ndarray, p: float) -> float:
    """Shift delta so that head weights w = g + delta fetch about a fraction p of random keys.

    Statistical model of the inputs only (not the indexer's arithmetic on data): for keys
    independent of the query, each head's dot product is roughly N(0, s^2), its ReLU has
    mean s/sqrt(2 pi) and variance s^2 (1/2 - 1/(2 pi)); the weighted sum is then roughly
    normal, and the fraction of non-negative sums is Phi(mean/std).  The ratio is
    monotone in delta (Cauchy-Schwarz), so bisection finds delta.
    """
    m_r = 1.0 / math.sqrt(2.0 * math.pi)
    v_r = 0.5 - 1.0 / (2.0 * math.pi)
    p = min(max(p, 1e-6), 1 - 1e-6)

    def rate(delta):
        w = g + delta
        return _phi(m_r * w.sum() / math.sqrt(v_r * float((w * w).sum()) + 1e-300))

    lo, hi = -50.0, 50.0
    for _ in range(100):
        mid = 0.5 * (lo + hi)
        if rate(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def _per_layer_rate(p_or: float, L: int) -> float:
    # layers draw independent keys, so the OR keeps 1 - prod(1 - p_l) of the entries
    return 1.0 - (1.0 - p_or) ** (1.0 / L)


CALIBRATION_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "fetch_calibration.json")


def _load_calibration():
    try:
        with open(CALIBRATION_FILE) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


_CALIBRATION = _load_calibration()


def model_target(wl: "Workload", b: int) -> float:
    """The target handed to the normal model for sequence b of wl: the calibrated value when the
    workload's name, seed, sequence id and wanted rate match an entry of the calibration file,
    the wanted rate itself otherwise."""
    cal = _CALIBRATION.get(wl.name)
    bid = wl._ids()[b]
    if cal and cal.get("seed") == wl.seed and bid < len(cal["target"]) and cal["target"][bid] == wl.fetch[b]:
        return float(cal["model_target"][bid])
    return float(wl.fetch[b])


@dataclass
class Inputs:
    """All inputs of one workload as CPU torch tensors in their storage dtypes."""
    wl: Workload
    seq_offsets: torch.Tensor            # int64 [B+1]
    h: torch.Tensor = None               # [L][B][d]                 dtype
    W_dq: torch.Tensor = None            # [L][r][d]   (out x in)    dtype
    W_iuq: torch.Tensor = None           # [L][n_h*d_I][r]           dtype
    W_w: torch.Tensor = None             # [L][n_h][d]               dtype
    w_target: torch.Tensor = None        # [L][B][n_h] float32 (what h was built to give)
    q: torch.Tensor = None               # [L][B][n_h][d_I]          dtype (stage-level draw)
    w: torch.Tensor = None               # [L][B][n_h] float32       (stage-level draw)
    K: torch.Tensor = None               # [L][sum S][d_I]           kdtype
    k_scale: torch.Tensor = None         # [L][sum S] float32 (fp8 keys only)
    planted: torch.Tensor = None         # [L][sum S] bool (which keys were planted)
    pool: torch.Tensor = None            # [sum S][row_bytes] uint8
    q_dec: torch.Tensor = None           # [B][tau][n_h][d_I]        dtype
    w_dec: torch.Tensor = None           # [B][tau][n_h] float32


def _draw_head_weights(wl: Workload, l: int, bid: int, p_or: float) -> np.ndarray:
    g = _rng(wl, "w", l, bid).standard_normal(wl.n_h)
    delta = _shift_for_rate(g, _per_layer_rate(p_or, wl.L))
    return (g + delta).astype(np.float32)


def plant_directions(wl: Workload, l: int) -> np.ndarray:
    """Unit planted direction of every head of layer l, [n_h][d_I] float64."""
    U = _rng(wl, "pdir", l).standard_normal((wl.n_h, wl.d_I))
    return U / np.linalg.norm(U, axis=1, keepdims=True)


def _draw_queries(wl: Workload, l: int, bid: int) -> np.ndarray:
    q = _rng(wl, "q", l, bid).standard_normal((wl.n_h, wl.d_I), dtype=np.float32)
    if wl.planted > 0:
        q += (math.sqrt(wl.d_I) * plant_directions(wl, l)).astype(np.float32)
    return q


def _keys_for(wl: Workload, l: int, b: int, bid: int, U: np.ndarray, w_b: np.ndarray):
    """Keys of one (layer, sequence): Gaussian N(0, 1/d_I) rows plus planted entries along
    v = normalise(sum_h w_h u_h) (U: the layer's planted directions, w_b the head weights)."""
    S = wl.S[b]
    K = _normal_rows(wl, "key", (l, bid), S, wl.d_I, 1.0 / math.sqrt(wl.d_I))
    planted = np.zeros(S, dtype=bool)
    if wl.planted > 0:
        # the planted positions are the sequence's (the same entries in every layer: an entry is
        # one compressed position of the context); the directions are the layer's
        prng = _rng(wl, "plant", bid)
        u = (w_b.astype(np.float64)[:, None] * U).sum(0)
        u /= np.linalg.norm(u) + 1e-300
        target = int(round(wl.planted * S))
        lo, hi = wl.planted_run
        while planted.sum() < target:
            run = int(prng.integers(lo, hi + 1))
            start = int(prng.integers(0, max(1, S - run + 1)))
            planted[start:start + run] = True
        idx = np.nonzero(planted)[0]
        n = _rng(wl, "plant", l, bid).standard_normal((idx.size, wl.d_I))
        n -= (n @ u)[:, None] * u[None, :]
        n /= np.linalg.norm(n, axis=1, keepdims=True) + 1e-300
        c = wl.planted_cos
        K[idx] = (c * u[None, :] + math.sqrt(1 - c * c) * n).astype(np.float32)
    return K, planted


def _encode_keys(K: np.ndarray, kdt: str):
    """Storage form of the keys: bf16/fp32 by rounding, or E4M3 codes with one fp32 scale per
    entry (scale = max |k| / 448, the largest finite E4M3 magnitude)."""
    if kdt != "fp8":
        return _cast(K, kdt), None
    Kt = torch.from_numpy(K)
    amax = Kt.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (Kt / scale[:, None]).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn)
    return codes, scale


def _hidden_for(wl: Workload, l: int, bid: int, QR, t: np.ndarray):
    """Hidden state h with h M = t exactly (before rounding h), for the constraint matrix M whose
    columns are W^w's (h W^w = the drawn head weights) and, with planted entries, W^DQ's row 0
    (c^Q[0] = PLANT_ALPHA).

    Construction from the weights alone: with M = Q R (Q orthonormal), h = h0 - Q Q^T h0 +
    Q R^{-T} t, where h0 ~ N(0, I).
    """
    Q, R = QR
    h0 = _rng(wl, "h", l, bid).standard_normal(wl.d)
    h = h0 - Q @ (Q.T @ h0) + Q @ np.linalg.solve(R.T, t.astype(np.float64))
    return h


def make_inputs(wl: Workload, parts=("proj", "score", "pool", "dec"), threads: int = _THREADS,
                pool_out: torch.Tensor = None) -> Inputs:
    """Draw the inputs of ``wl``.

    parts: "proj" (h and projection weights), "score" (stage-level q, w and the keys),
    "pool" (cold-pool KV rows), "dec" (decode-step queries of the Lightning Indexer).
    Keys are always drawn when "score" or "proj" is requested.  pool_out: an existing uint8
    [sum S][row_bytes] host tensor (e.g. mapped page-locked memory) to fill in place.
    """
    parts = set(parts)
    ids = wl._ids()
    offs = wl.seq_offsets
    inp = Inputs(wl=wl, seq_offsets=torch.from_numpy(offs.copy()))
    L, B = wl.L, wl.B

    # stage-level queries and head weights (also give the planted direction)
    qs = np.zeros((L, B, wl.n_h, wl.d_I), dtype=np.float32)
    ws = np.zeros((L, B, wl.n_h), dtype=np.float32)
    for l in range(L):
        for b in range(B):
            qs[l, b] = _draw_queries(wl, l, ids[b])
            ws[l, b] = _draw_head_weights(wl, l, ids[b], model_target(wl, b))
    q_t = _cast(qs, wl.dtype)
    if "score" in parts or "proj" in parts:
        inp.q = q_t
        inp.w = torch.from_numpy(ws)
        Us = [plant_directions(wl, l) for l in range(L)] if wl.planted > 0 else [None] * L
        T = wl.total_S
        K_all = torch.empty((L, T, wl.d_I), dtype=DTYPES[wl.kdtype])
        sc_all = torch.empty((L, T), dtype=torch.float32) if wl.kdtype == "fp8" else None
        pl_all = torch.zeros((L, T), dtype=torch.bool)

        def job(lb):
            l, b = lb
            K, pl = _keys_for(wl, l, b, ids[b], Us[l], ws[l, b])
            Kt, sc = _encode_keys(K, wl.kdtype)
            s0, s1 = int(offs[b]), int(offs[b + 1])
            K_all[l, s0:s1] = Kt
            if sc is not None:
                sc_all[l, s0:s1] = sc
            pl_all[l, s0:s1] = torch.from_numpy(pl)

        for lb in [(l, b) for l in range(L) for b in range(B)]:
            job(lb)
        inp.K, inp.k_scale, inp.planted = K_all, sc_all, pl_all

    if "proj" in parts:
        d, r, nq = wl.d, wl.r, wl.n_h * wl.d_I
        W_dq = np.empty((L, r, d), dtype=np.float32)
        W_iuq = np.empty((L, nq, r), dtype=np.float32)
        W_w = np.empty((L, wl.n_h, d), dtype=np.float32)
        planted = wl.planted > 0
        beta = math.sqrt(wl.d_I) / PLANT_ALPHA
        for l in range(L):
            _normal_rows(wl, "wdq", (l,), r, d, 1.0 / math.sqrt(d), out=W_dq[l])
            _normal_rows(wl, "wiuq", (l,), nq, r, 1.0 / math.sqrt(r), out=W_iuq[l])
            _normal_rows(wl, "ww", (l,), wl.n_h, d, 1.0 / math.sqrt(d), out=W_w[l])
            if planted:
                W_iuq[l, :, 0] = (beta * plant_directions(wl, l)).reshape(nq)
        inp.W_dq, inp.W_iuq, inp.W_w = _cast(W_dq, wl.dtype), _cast(W_iuq, wl.dtype), _cast(W_w, wl.dtype)
        # h is built against the *stored* (rounded) weights so that h W^w (and c^Q[0]) land on the targets
        hs = np.zeros((L, B, d), dtype=np.float64)
        for l in range(L):
            M = inp.W_w[l].double().numpy()             # [n_h][d] = (W^w)^T
            if planted:
                M = np.concatenate([M, inp.W_dq[l, :1].double().numpy()], axis=0)
            QR = np.linalg.qr(M.T)                      # d x (n_h [+ 1])
            for b in range(B):
                t = np.concatenate([ws[l, b], [PLANT_ALPHA]]) if planted else ws[l, b]
                hs[l, b] = _hidden_for(wl, l, ids[b], QR, t)
        inp.h = _cast(hs, wl.dtype)
        inp.w_target = torch.from_numpy(ws.copy())

    if "pool" in parts:
        T = wl.total_S
        pool = pool_out if pool_out is not None else torch.empty((T, wl.row_bytes), dtype=torch.uint8)

        def pjob(b):
            s0, s1 = int(offs[b]), int(offs[b + 1])
            words = _rng(wl, "pool", ids[b]).integers(0, 2 ** 32, size=((s1 - s0) * wl.row_bytes // 4,),
                                                      dtype=np.uint32)
            pool[s0:s1] = torch.from_numpy(words.view(np.uint8).reshape(s1 - s0, wl.row_bytes))

        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(pjob, range(B)))
        inp.pool = pool

    if "dec" in parts:
        qd = np.zeros((B, wl.tau, wl.n_h, wl.d_I), dtype=np.float32)
        wd = np.zeros((B, wl.tau, wl.n_h), dtype=np.float32)
        for b in range(B):
            qd[b] = _rng(wl, "qdec", ids[b]).standard_normal((wl.tau, wl.n_h, wl.d_I), dtype=np.float32)
            wd[b] = _rng(wl, "wdec", ids[b]).standard_normal((wl.tau, wl.n_h), dtype=np.float32)
        inp.q_dec = _cast(qd, wl.dtype)
        inp.w_dec = torch.from_numpy(wd)
    return inp


def random_fetch_list(wl: Workload, rate: float, seed: int = 0):
    """A seeded ascending fetched-entry list per sequence (stage-level input of the
    gather and the decode-step Top-k): idx [sum S] int32 (segment b at seq_offsets[b],
    first count[b] slots used) and count [B] int32."""
    offs = wl.seq_offsets
    idx = np.full(wl.total_S, -1, dtype=np.int32)
    cnt = np.zeros(wl.B, dtype=np.int32)
    ids = wl._ids()
    for b in range(wl.B):
        S = wl.S[b]
        rng = np.random.default_rng([wl.seed, 99, seed, ids[b]])
        sel = np.nonzero(rng.random(S) < rate)[0].astype(np.int32)
        idx[offs[b]:offs[b] + sel.size] = sel
        cnt[b] = sel.size
    return torch.from_numpy(idx), torch.from_numpy(cnt)


def golden_logits(S, tau: int = 64, Lc: int = 21, seed: int = 2024, planted_frac: float = 0.012,
                  delta: float = 6.0, agree: float = 0.8, spurious: int = 10):
    """Raw indexer logits of one future window for the golden-label step, z [tau][Lc][T] float32,
    and seq_offsets [B+1] int64 (entry s of sequence b at column seq_offsets[b] + s).

    Background logits are N(0, 1).  Each sequence has a fraction `planted_frac` of relevant entries
    in contiguous runs of 8-64; a relevant entry gets +delta + N(0, 0.5) in each (token, layer)
    row with probability `agree`, so most layers agree on it.  Every row also lifts `spurious`
    random entries by delta: peaks that one layer sees and the others do not.  With the defaults
    the softmax mass of a row is about 70 % relevant entries, and the cross-layer vote keeps a few
    hundred entries per sequence (the pages report 100-1,000 golden entries per window).
    """
    S = [int(x) for x in S]
    offs = np.zeros(len(S) + 1, dtype=np.int64)
    offs[1:] = np.cumsum(S)
    T = int(offs[-1])
    g = torch.Generator().manual_seed(seed)
    z = torch.randn((tau, Lc, T), generator=g, dtype=torch.float32)
    rng = np.random.default_rng(seed)
    planted = []
    for b, n in enumerate(S):
        want = int(planted_frac * n)
        got = []
        while sum(len(r) for r in got) < want and n > 64:
            start = int(rng.integers(0, n - 64))
            got.append(np.arange(start, start + int(rng.integers(8, 65))))
        if got:
            planted.append(offs[b] + np.unique(np.concatenate(got)))
    planted = torch.from_numpy(np.concatenate(planted)) if planted else torch.zeros(0, dtype=torch.int64)
    if planted.numel():
        on = torch.rand((tau, Lc, planted.numel()), generator=g) < agree
        lift = delta + 0.5 * torch.randn((tau, Lc, planted.numel()), generator=g)
        z[:, :, planted] += torch.where(on, lift, torch.zeros_like(lift))
    if T and spurious:
        cols = torch.randint(0, T, (tau, Lc, spurious), generator=g)
        z.scatter_add_(2, cols, torch.full((tau, Lc, spurious), delta))
    return z, torch.from_numpy(offs)

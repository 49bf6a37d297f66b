"""Agreement rules between the CUDA path and the CPU oracle.

Fetch decisions and index lists must be bit-exact, except entries whose oracle score lies
within 2e-3 of the threshold (after the sigmoid) in a layer that could decide the OR.  Sigmoid
scores agree within 2e-3 absolute.  Lightning-Indexer scores (no sigmoid) agree within a
bound derived from fp32 accumulation: |dy| <= 2^-22 (d_I + n_h + 2) sum_h |w_h| A_h, where
A_h = scale * sum_e |q_h[e]| |K[e]| bounds every partial sum of the dot product; entries
whose oracle score is within that bound of the k-th score may swap in or out of the Top-k.
"""
import numpy as np
import torch

import oracle

SIGMOID_TOL = 2e-3


def or_exempt(I_oracle: np.ndarray, thr: float = 0.5, tol: float = SIGMOID_TOL) -> np.ndarray:
    """Entries whose OR decision could flip within the tolerance: no layer is clearly above
    the threshold and at least one layer is within tol of it."""
    clearly_in = (I_oracle >= thr + tol).any(axis=0)
    clearly_out = (I_oracle < thr - tol).all(axis=0)
    return ~(clearly_in | clearly_out)


def check_select(mask_gpu, idx_gpu, cnt_gpu, I_gpu, ref, offs, thr=0.5, what=""):
    """mask_gpu [T] uint8, idx_gpu [T], cnt_gpu [B], I_gpu [L][T] or None; ref: oracle.score dict."""
    offs = np.asarray(offs)
    B = offs.size - 1
    ex = or_exempt(ref["I"], thr)
    bad = (mask_gpu != ref["mask"]) & ~ex
    assert not bad.any(), f"{what}: {bad.sum()} fetch decisions differ outside the threshold band " \
                          f"(first at {np.nonzero(bad)[0][:5]})"
    for b in range(B):
        seg = mask_gpu[offs[b]:offs[b + 1]]
        assert cnt_gpu[b] == seg.sum(), f"{what}: count[{b}] {cnt_gpu[b]} != popcount {seg.sum()}"
        got = idx_gpu[offs[b]:offs[b] + cnt_gpu[b]]
        assert np.array_equal(got, np.nonzero(seg)[0]), f"{what}: idx list of sequence {b} is not the ascending mask"
    if I_gpu is not None:
        err = np.abs(I_gpu.astype(np.float64) - ref["I"])
        assert err.max() <= SIGMOID_TOL, f"{what}: sigmoid score error {err.max()}"
    return int(ex.sum()), int(((mask_gpu != ref["mask"]) & ex).sum())


def keys_as_float(K_rows: torch.Tensor, scale_rows) -> torch.Tensor:
    Kf = K_rows.float()
    if scale_rows is not None:
        Kf = Kf * scale_rows.float()[:, None]
    return Kf


def li_tolerance(q_dec_bi: torch.Tensor, w_dec_bi: torch.Tensor, Kf: torch.Tensor) -> np.ndarray:
    """Per-candidate bound on the fp32 error of y for one query.
    q_dec_bi [n_h][d_I], w_dec_bi [n_h], Kf [F][d_I] decoded (scaled) keys."""
    n_h, d_I = q_dec_bi.shape
    A = torch.abs(q_dec_bi.double()) @ torch.abs(Kf.double()).T     # [n_h][F]
    mag = (torch.abs(w_dec_bi.double())[:, None] * A).sum(0)        # [F]
    return (2.0 ** -22) * (d_I + n_h + 2) * mag.numpy()


def check_topk_query(gi, gs, y_or, s_list, tol, k, what=""):
    """gi/gs: GPU Top-k indices and scores of one query; y_or: oracle scores of the fetched slots
    (aligned with s_list, the fetched entries); tol: per-slot bound."""
    F = len(s_list)
    n = min(k, F)
    assert (gi[n:] == -1).all() and np.isneginf(gs[n:]).all(), f"{what}: padding wrong"
    sel = gi[:n]
    assert len(set(sel.tolist())) == n, f"{what}: duplicate entries"
    pos = {int(s): j for j, s in enumerate(s_list)}
    assert all(int(s) in pos for s in sel), f"{what}: selected entry not in the fetched set"
    slots = np.array([pos[int(s)] for s in sel], dtype=np.int64)
    # scores of the selected slots
    err = np.abs(gs[:n].astype(np.float64) - y_or[slots])
    assert (err <= tol[slots] + 1e-30).all(), f"{what}: score error {err.max()} above bound {tol[slots].max()}"
    # ordering by the GPU's own scores: non-increasing, equal scores by ascending entry
    for a in range(n - 1):
        assert gs[a] > gs[a + 1] or (gs[a] == gs[a + 1] and sel[a] < sel[a + 1]), f"{what}: order at {a}"
    if F > k:
        order = np.lexsort((np.asarray(s_list), -y_or))
        yk = y_or[order[k - 1]]
        tmax = float(tol.max())
        chosen = np.zeros(F, dtype=bool)
        chosen[slots] = True
        # an entry more than 2 tmax above (below) the k-th oracle score cannot be overtaken
        # by (cannot overtake) the entries on the other side, whatever the rounding
        must_in = y_or > yk + 2 * tmax
        must_out = y_or < yk - 2 * tmax
        assert chosen[must_in].all(), f"{what}: {(~chosen[must_in]).sum()} clear Top-k entries missing"
        assert not chosen[must_out].any(), f"{what}: {chosen[must_out].sum()} clear non-Top-k entries selected"
        return int((~must_in & ~must_out).sum())
    return 0


def check_project(h, W_dq, W_iuq, W_w, n_h, d_I, q_gpu, w_gpu, c_gpu, what=""):
    """Stage 1 against the oracle, in two exact halves (all tensors on the CPU, [L][B]... layout).

    c = h W^DQ rounded to the storage type: the GPU's fp32 sum and the oracle's exact sum may round
    to neighbouring values, |dc| <= ulp + 2^-22 d sum|h W|.  A neighbour of c moves q by far more
    than one ulp of q where q cancels, so q is checked against the oracle's second projection of
    the GPU's own c (identity as W^DQ makes the oracle's first projection an exact copy of c):
    |dq| <= ulp + 2^-22 r sum|c W^IUQ|.  w = h W^w in fp32: |dw| <= 2^-22 d sum|h W^w|.
    """
    L, B, d = h.shape
    r = W_dq.shape[1]
    bf = h.dtype == torch.bfloat16
    ulp = (lambda a, b: torch.maximum(a.abs(), b.abs()) * 2.0 ** -7) if bf else (lambda a, b: torch.zeros_like(a))
    q_ref, w_ref, c_ref = oracle.project(h, W_dq, W_iuq, W_w, n_h, d_I, want_c=True)
    h64 = h.double()
    wb = (2.0 ** -22) * d * torch.einsum("lbi,lhi->lbh", h64.abs(), W_w.double().abs())
    assert ((w_gpu.double() - w_ref.double()).abs() <= wb).all(), f"{what}: w"
    cb = (2.0 ** -22) * d * torch.einsum("lbi,lji->lbj", h64.abs(), W_dq.double().abs())
    dc = (c_gpu.double() - c_ref.double()).abs()
    assert (dc <= ulp(c_gpu.double(), c_ref.double()) * 1.0001 + cb).all(), f"{what}: c"
    if bf:  # neighbours only where the exact c lies near a rounding boundary
        assert (dc > 0).double().mean() < 0.15, f"{what}: too many c differ"
    eye = torch.eye(r, dtype=h.dtype).expand(L, r, r).contiguous()
    q2, _ = oracle.project(c_gpu.contiguous(), eye, W_iuq, torch.zeros((L, n_h, r), dtype=h.dtype), n_h, d_I)
    qb = (2.0 ** -22) * r * torch.einsum("lbj,loj->lbo", c_gpu.double().abs(), W_iuq.double().abs())
    dq = (q_gpu.double() - q2.double()).reshape(qb.shape).abs()
    assert (dq <= ulp(q_gpu.double(), q2.double()).reshape(qb.shape) * 1.0001 + qb).all(), f"{what}: q"
    if bf:
        assert (dq > 0).double().mean() < 0.05, f"{what}: too many q differ"

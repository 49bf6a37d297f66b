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
    if bf:
        # a stored c may differ from the oracle's only as the other side of a rounding boundary
        # that the exact sum lies within the fp32 bound of: the GPU's fp32 sum s is within cb of
        # the exact sum x and rounds to the other neighbour, so the midpoint between the two
        # neighbours lies between x and s
        c_exact = torch.einsum("lbi,lji->lbj", h64, W_dq.double())
        _near_boundary(c_exact, c_ref.double(), c_gpu.double(), cb, f"{what}: c")
    eye = torch.eye(r, dtype=h.dtype).expand(L, r, r).contiguous()
    q2, _ = oracle.project(c_gpu.contiguous(), eye, W_iuq, torch.zeros((L, n_h, r), dtype=h.dtype), n_h, d_I)
    qb = (2.0 ** -22) * r * torch.einsum("lbj,loj->lbo", c_gpu.double().abs(), W_iuq.double().abs())
    dq = (q_gpu.double() - q2.double()).reshape(qb.shape).abs()
    assert (dq <= ulp(q_gpu.double(), q2.double()).reshape(qb.shape) * 1.0001 + qb).all(), f"{what}: q"
    if bf:
        q_exact = torch.einsum("lbj,loj->lbo", c_gpu.double(), W_iuq.double())
        _near_boundary(q_exact, q2.double().reshape(qb.shape), q_gpu.double().reshape(qb.shape), qb, f"{what}: q")


def _near_boundary(exact, ref, got, bound, what):
    """Where got != ref (both rounded values), the rounding boundary between them (their midpoint)
    is within bound of the exact value (1e-12 relative slack for the double sums)."""
    diff = got != ref
    if not bool(diff.any()):
        return
    mid = (ref[diff] + got[diff]) / 2
    gap = (exact[diff] - mid).abs()
    lim = bound[diff] * 1.0001 + exact[diff].abs() * 1e-12
    assert (gap <= lim).all(), f"{what}: a value differs away from a rounding boundary"


# ------------------------------------------------------------------------------ training step

def exact_train_case(dt, kdt, L=2, S=(300, 0, 129, 517), d=512, r=256, n_h=64, d_I=128, seed=7, h_nz=24,
                     wiuq_nz=8, label_rate=0.25):
    """Inputs of one indexer training step on which every forward quantity is exact in fp32 on the
    GPU, in bf16/E4M3 storage and in the oracle's double: h has h_nz entries of +-1 per (layer,
    sequence), W^DQ entries are -1, 0 or 1 (so |c| <= h_nz), each W^IUQ row has wiuq_nz entries +-1
    (so q is an integer of magnitude <= h_nz * wiuq_nz <= 256, exact in bf16), W^w entries are
    {-1, 0, 1} / 32 and keys {-1, 0, 1} times a power of two (bf16 values 2^-6; E4M3 codes with
    per-entry scales 2^-6 or 2^-7).  The head dot products, the ReLU gates and the logits are then
    the same on both sides (`train_bounds` asserts the premise), so the two sides differ only by the
    fp32 evaluation of the loss derivative and the fp32 sums of the gradients.

    dt: torch.float32 or torch.bfloat16 (h and weights); kdt: the key type (float32, bfloat16 or
    float8_e4m3fn).  Returns (h, [W_dq, W_iuq, W_w], K, k_scale, labels, seq_offsets, n_h, d_I).
    """
    rng = np.random.default_rng(seed)
    B = len(S)
    nq = n_h * d_I
    offs = np.concatenate([[0], np.cumsum(S)]).astype(np.int64)
    T = int(offs[-1])
    h = np.zeros((L, B, d))
    for l in range(L):
        for b in range(B):
            pos = rng.choice(d, h_nz, replace=False)
            h[l, b, pos] = rng.choice([-1.0, 1.0], h_nz)
    W_dq = rng.integers(-1, 2, size=(L, r, d)).astype(np.float64)
    W_iuq = np.zeros((L, nq, r))
    for l in range(L):
        cols = np.argsort(rng.random((nq, r)), axis=1)[:, :wiuq_nz]
        W_iuq[l, np.arange(nq)[:, None], cols] = rng.choice([-1.0, 1.0], (nq, wiuq_nz))
    W_w = rng.integers(-1, 2, size=(L, n_h, d)) / 32.0
    codes = rng.integers(-1, 2, size=(L, T, d_I)).astype(np.float64)
    labels = (rng.random(T) < label_rate).astype(np.uint8)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dt)
    if kdt == torch.float8_e4m3fn:
        K = torch.from_numpy(codes.astype(np.float32)).to(kdt)
        k_scale = torch.from_numpy(rng.choice([2.0 ** -6, 2.0 ** -7], (L, T)).astype(np.float32))
    else:
        K = torch.from_numpy((codes * 2.0 ** -6).astype(np.float32)).to(kdt)
        k_scale = None
    return (t(h), [t(W_dq), t(W_iuq), t(W_w)], K, k_scale, torch.from_numpy(labels), torch.from_numpy(offs),
            n_h, d_I)


def _focal_terms(x, y, gamma, alpha):
    """Per-entry focal loss and its derivative in the logit (binary cross-entropy at gamma = 0,
    alpha < 0), in double."""
    p = 1.0 / (1.0 + np.exp(-x))
    pt = np.where(y, p, 1.0 - p)
    at = np.ones_like(x) if alpha < 0 else np.where(y, alpha, 1.0 - alpha)
    lpt = np.where(y, -np.log1p(np.exp(-x)), -np.log1p(np.exp(x)))
    q1 = 1.0 - pt
    loss = -at * q1 ** gamma * lpt
    if gamma == 0.0:
        dl = at * np.where(y, p - 1.0, p)
    else:
        dl = at * (gamma * q1 ** (gamma - 1.0) * lpt * pt * q1 - q1 ** gamma * q1) * np.where(y, 1.0, -1.0)
    return loss, dl, at


def train_bounds(case, gamma=0.0, alpha=-1.0):
    """Per-element bounds on |GPU - oracle| for the loss and the three weight gradients of one
    training step on exact inputs (`exact_train_case`).

    The forward is exact on both sides (asserted here), so the differences are:
      * the loss derivative g_s = dl/dx / N, evaluated in fp32 from an exact logit: its absolute
        error is below 2^-18 a_t / N for binary cross-entropy and the focal loss with gamma <= 2
        (a few ulps of each fp32 factor; |dl/dx| <= a_t); G_sh = g_s w_h scale_s is two more fp32
        roundings, and the tensor-core path splits it into bf16 parts hi + lo (|G - hi - lo| <=
        2^-18 |G|): 2^-17 |G| covers both;
      * every fp32 sum, in whatever order (register tiles, warp shuffles, atomics, tensor-core
        accumulation): at most 2^-22 m sum |term|, m the number of its nonzero terms (four times the
        classical m 2^-24 bound; adding an exact zero rounds nothing, and these inputs are sparse);
      * the errors of dq and dw carried through dc = dq W^IUQ and the outer products over sequences.
    Returns dict with the exact forward's magnitudes and the bounds E_loss, E_g_Wdq, E_g_Wiuq, E_g_Ww.
    """
    h, (W_dq, W_iuq, W_w), K, k_scale, labels, offs, n_h, d_I = case
    L, B, d = h.shape
    r = W_dq.shape[1]
    nq = n_h * d_I
    offs = np.asarray(offs)
    T = int(offs[-1])
    N = float(L * T)
    H = h.double().numpy()
    Wdq, Wiuq, Ww = W_dq.double().numpy(), W_iuq.double().numpy(), W_w.double().numpy()
    Kraw = K.float().double().numpy()                                  # stored values (E4M3: the codes)
    sc = k_scale.double().numpy() if k_scale is not None else np.ones((L, T))
    c = np.einsum("lbi,lji->lbj", H, Wdq)
    q = np.einsum("lbj,loj->lbo", c, Wiuq)
    w = np.einsum("lbi,lhi->lbh", H, Ww)
    assert np.all(np.abs(c) <= 256) and np.all(c == np.round(c)), "premise: c exact in bf16"
    assert np.all(np.abs(q) <= 256) and np.all(q == np.round(q)), "premise: q exact in bf16"
    y = np.asarray(labels).astype(bool)
    u22 = 2.0 ** -22
    E_dq = np.zeros((L, B, nq))
    A_dq = np.zeros((L, B, nq))   # |dq| + E_dq
    E_dw = np.zeros((L, B, n_h))
    A_dw = np.zeros((L, B, n_h))
    loss_abs = 0.0
    loss = 0.0
    for l in range(L):
        for b in range(B):
            s0, s1 = int(offs[b]), int(offs[b + 1])
            S = s1 - s0
            if S == 0:
                continue
            Kr = Kraw[l, s0:s1]
            scs = sc[l, s0:s1]
            qh = q[l, b].reshape(n_h, d_I)
            a = (Kr @ qh.T) * scs[:, None]                            # [S][n_h], exact
            relu = np.maximum(a, 0.0)
            wx = np.abs(w[l, b])[None, :] * relu
            assert wx.sum(1).max() < 2.0 ** 12, "premise: logits exact in fp32"
            x = (w[l, b][None, :] * relu).sum(1)
            ls, dl, at = _focal_terms(x, y[s0:s1], gamma, alpha)
            loss += ls.sum()
            loss_abs += np.abs(ls).sum()
            g = dl / N
            dg = 2.0 ** -18 * at / N
            pos = a > 0
            G = g[:, None] * w[l, b][None, :] * scs[:, None] * pos
            dG = (dg[:, None] * np.abs(w[l, b])[None, :] * scs[:, None] + 2.0 ** -17 * np.abs(G)) * pos
            aK = np.abs(Kr)
            m = (G != 0).T.astype(np.float64) @ (aK > 0)              # nonzero terms of each dq sum
            e = dG.T @ aK + u22 * m * (np.abs(G).T @ aK)              # [n_h][d_I]
            E_dq[l, b] = e.reshape(nq)
            A_dq[l, b] = np.abs(G.T @ Kr).reshape(nq) + E_dq[l, b]
            mw = (g != 0).astype(np.float64) @ (relu > 0)
            E_dw[l, b] = dg @ relu + u22 * mw * (np.abs(g) @ relu)
            A_dw[l, b] = np.abs(g @ relu) + E_dw[l, b]
    nz = lambda x: (x != 0).astype(np.float64)
    aW = np.abs(Wiuq)
    m_dc = np.einsum("lbo,loj->lbj", nz(A_dq), nz(Wiuq))
    E_dc = np.einsum("lbo,loj->lbj", E_dq, aW) + u22 * m_dc * np.einsum("lbo,loj->lbj", A_dq, aW)
    A_dc = np.einsum("lbo,loj->lbj", A_dq, aW) + E_dc                  # a bound on |dc| + its error
    ac, aH = np.abs(c), np.abs(H)
    m_iuq = np.einsum("lbo,lbj->loj", nz(A_dq), nz(c))
    m_wdq = np.einsum("lbj,lbi->lji", nz(A_dc), nz(H))
    m_ww = np.einsum("lbh,lbi->lhi", nz(A_dw), nz(H))
    E_iuq = np.einsum("lbo,lbj->loj", E_dq, ac) + u22 * m_iuq * np.einsum("lbo,lbj->loj", A_dq, ac)
    E_wdq = np.einsum("lbj,lbi->lji", E_dc, aH) + u22 * m_wdq * np.einsum("lbj,lbi->lji", A_dc, aH)
    E_ww = np.einsum("lbh,lbi->lhi", E_dw, aH) + u22 * m_ww * np.einsum("lbh,lbi->lhi", A_dw, aH)
    return {"loss": loss / N, "E_loss": 2.0 ** -20 * loss_abs / N + 1e-15,
            "E_g_Wdq": E_wdq, "E_g_Wiuq": E_iuq, "E_g_Ww": E_ww}


def check_train(loss, grads, ref, bounds, what=""):
    """loss (float) and grads (g_Wdq, g_Wiuq, g_Ww as float64 arrays) of the CUDA path against the
    oracle's `ref`, element by element within `bounds` (train_bounds)."""
    assert abs(loss - ref["loss"]) <= bounds["E_loss"], f"{what}: loss {loss} vs {ref['loss']}"
    for got, key in zip(grads, ("g_Wdq", "g_Wiuq", "g_Ww")):
        assert np.isfinite(got).all(), f"{what}: {key} not finite"
        err = np.abs(got - ref[key])
        bad = err > bounds["E_" + key]
        if bad.any():
            i = np.unravel_index(np.argmax(err - bounds["E_" + key]), err.shape)
            raise AssertionError(f"{what}: {key}: {int(bad.sum())} of {bad.size} elements outside their bound; "
                                 f"worst at {i}: got {got[i]!r}, oracle {ref[key][i]!r}, bound {bounds['E_' + key][i]!r}")

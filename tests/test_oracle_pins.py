"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each ``pin_*`` function checks one fact fixed by the pages' formulas or by mathematics:
a hand-worked example (tests/golden/hand_example.json), closed forms, special cases that
reduce to a library routine (numpy dot/lexsort, torch dtype casts), invariants, and an
exhaustive enumeration on tiny inputs.  ``test_mutants_are_caught`` compiles deliberately
broken copies of the oracle source and checks that the pins reject every one of them.
"""
import itertools
import json
import math
import os
import shutil
import subprocess
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_example.json")


def _t(a, dt=torch.float32):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(dt)


def _offs(*S):
    return np.concatenate([[0], np.cumsum(S)]).astype(np.int64)


# ------------------------------------------------------------------ storage formats

def pin_bf16_matches_torch_cast():
    rng = np.random.default_rng(0)
    normal = rng.standard_normal(20000).astype(np.float32)
    tiny = (rng.standard_normal(2000) * 1e-39).astype(np.float32)    # bf16 subnormals
    with np.errstate(over="ignore"):  # the near-overflow draws include some that round to +-inf
        big = (rng.standard_normal(2000) * 1e38).astype(np.float32)
    x = np.concatenate([
        normal,
        tiny,
        big,                                                         # near overflow
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.3895314e38, 3.39e38, 1e-45,
                  -1.00390625, 2.0 ** -126, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135], dtype=np.float32),
    ])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_bits(x.astype(np.float64))
    assert np.array_equal(got, want)


def pin_bf16_nearest_even_exact():
    """For reals that are not float32 values, the result is the nearer bf16 neighbour
    (exact rational arithmetic), ties to the even significand."""
    rng = np.random.default_rng(1)
    xs = list(rng.standard_normal(300) * 10.0 ** rng.integers(-30, 30, 300))
    xs += [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -40]  # tie, tie, above tie
    bits = oracle.bf16_bits(np.array(xs))

    def value(b):  # bf16 bits are the top half of a binary32
        return Fraction(float((np.array([b & 0xFFFF], dtype=np.uint32) << 16).view(np.float32)[0]))

    for x, b in zip(xs, bits):
        b = int(b)
        val, X = value(b), Fraction(x)
        for nb in (b + 1, b - 1):           # the neighbouring bf16 values (same sign side)
            nv = value(nb)
            assert abs(X - val) <= abs(X - nv)
            if abs(X - val) == abs(X - nv):
                assert b % 2 == 0


def pin_e4m3_matches_torch_cast():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = oracle.e4m3_decode(codes)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def pin_sigmoid_closed_forms():
    assert oracle.sigmoid(0.0) == 0.5
    assert abs(oracle.sigmoid(math.log(3.0)) - 0.75) < 1e-15
    for x in (0.3, 1.7, 5.0, 20.0):
        assert abs(oracle.sigmoid(x) + oracle.sigmoid(-x) - 1.0) < 1e-15


# ------------------------------------------------------------------ projections

def pin_project_matches_library_matmul():
    """Non-square random shapes (d != r, n_h != d_I): c = h W^DQ, q = c W^IUQ, w = h W^w
    against numpy matmul in float64 with the same fp32 storage rounding of c and q."""
    rng = np.random.default_rng(2)
    L, B, d, r, n_h, d_I = 2, 3, 24, 10, 3, 5
    h = rng.standard_normal((L, B, d)).astype(np.float32)
    Wdq = rng.standard_normal((L, r, d)).astype(np.float32)
    Wiuq = rng.standard_normal((L, n_h * d_I, r)).astype(np.float32)
    Ww = rng.standard_normal((L, n_h, d)).astype(np.float32)
    q, w, c = oracle.project(_t(h), _t(Wdq), _t(Wiuq), _t(Ww), n_h, d_I, want_c=True)
    for l in range(L):
        c_ref = (h[l].astype(np.float64) @ Wdq[l].T.astype(np.float64)).astype(np.float32)
        q_ref = (c_ref.astype(np.float64) @ Wiuq[l].T.astype(np.float64)).astype(np.float32)
        w_ref = (h[l].astype(np.float64) @ Ww[l].T.astype(np.float64)).astype(np.float32)
        np.testing.assert_array_max_ulp(c[l].numpy(), c_ref, maxulp=1)
        np.testing.assert_array_max_ulp(q[l].reshape(B, -1).numpy(), q_ref, maxulp=1)
        np.testing.assert_array_max_ulp(w[l].numpy(), w_ref, maxulp=1)


def pin_project_integer_exact_bf16():
    """Small integers: every sum is an exact integer below 256, so bf16 storage is exact
    and the result must equal the integer matmul."""
    rng = np.random.default_rng(3)
    L, B, d, r, n_h, d_I = 1, 2, 6, 4, 2, 3
    h = rng.integers(-2, 3, (L, B, d))
    Wdq = rng.integers(-1, 2, (L, r, d))
    Wiuq = rng.integers(-1, 2, (L, n_h * d_I, r))
    Ww = rng.integers(-2, 3, (L, n_h, d))
    q, w = oracle.project(_t(h, torch.bfloat16), _t(Wdq, torch.bfloat16), _t(Wiuq, torch.bfloat16),
                          _t(Ww, torch.bfloat16), n_h, d_I)
    c_ref = h[0] @ Wdq[0].T
    assert np.abs(c_ref).max() < 256
    q_ref = c_ref @ Wiuq[0].T
    assert np.array_equal(q[0].float().reshape(B, -1).numpy(), q_ref.astype(np.float32))
    assert np.array_equal(w[0].numpy(), (h[0] @ Ww[0].T).astype(np.float32))


def pin_project_bf16_storage_points():
    """Integer inputs whose sums need more than bf16's 8 significant bits: c must be stored
    in bf16 (rounded once, nearest-even) before the second projection, and q rounded once
    more.  Every sum is an exact integer in fp32, so torch's single fp32 -> bf16 cast gives
    the expected values."""
    rng = np.random.default_rng(15)
    L, B, d, r, n_h, d_I = 1, 3, 16, 8, 2, 3
    h = rng.integers(-20, 21, (L, B, d))
    Wdq = rng.integers(-5, 6, (L, r, d))
    Wiuq = rng.integers(-3, 4, (L, n_h * d_I, r))
    Ww = rng.integers(-5, 6, (L, n_h, d))
    bf = torch.bfloat16
    q, w, c = oracle.project(_t(h, bf), _t(Wdq, bf), _t(Wiuq, bf), _t(Ww, bf), n_h, d_I, want_c=True)
    c_int = h[0] @ Wdq[0].T
    assert np.abs(c_int).max() > 256                       # rounding really happens
    c_ref = torch.from_numpy(c_int.astype(np.float32)).to(bf)
    assert torch.equal(c[0].view(torch.int16), c_ref.view(torch.int16))
    q_int = c_ref.double().numpy() @ Wiuq[0].T
    assert np.abs(q_int).max() < 2 ** 24
    q_ref = torch.from_numpy(q_int.astype(np.float32)).to(bf)
    assert torch.equal(q[0].reshape(B, -1).view(torch.int16), q_ref.view(torch.int16))
    assert np.array_equal(w[0].numpy(), (h[0] @ Ww[0].T).astype(np.float32))
    q2, _ = oracle.project(_t(h, bf), _t(Wdq, bf), _t(Wiuq, bf), _t(Ww, bf), n_h, d_I)
    assert torch.equal(q2.view(torch.int16), q.view(torch.int16))


def pin_project_identity_weights():
    """W^DQ = I (r = d) and W^IUQ = I make q a copy of h rounded to bf16."""
    rng = np.random.default_rng(4)
    d, n_h, d_I = 8, 2, 4
    h = rng.standard_normal((1, 2, d))
    q, w = oracle.project(_t(h, torch.bfloat16), _t(np.eye(d)[None], torch.bfloat16),
                          _t(np.eye(d)[None], torch.bfloat16), _t(np.eye(d)[None, :n_h], torch.bfloat16),
                          n_h, d_I)
    hb = _t(h, torch.bfloat16)
    assert torch.equal(q.reshape(1, 2, d), hb)
    assert torch.equal(w, hb[..., :n_h].float())


# ------------------------------------------------------------------ index score / fetch

def pin_hand_example():
    with open(GOLD) as f:
        g = json.load(f)
    q = _t(g["q"])[:, None]                     # [L][B=1][n_h][d_I]
    w = _t(g["w"])[:, None]
    K = _t(g["K"])                              # [L][S][d_I]
    offs = _offs(K.shape[1])
    out = oracle.score(q, w, K, None, offs, 0.5)
    assert np.array_equal(out["x"], np.array(g["x"], dtype=np.float64))
    for l in range(2):
        for s in range(6):
            assert out["I"][l, s] == pytest.approx(g["sigmoid"][str(g["x"][l][s])], abs=1e-15)
    assert out["mask"].tolist() == g["mask_or"]
    assert out["idx"][:out["count"][0]].tolist() == g["idx"]
    assert oracle.score(q, w, K, None, offs, 0.75)["mask"].tolist() == g["mask_or_thr075"]
    # decode-step Lightning Indexer over the fetched set with layer-0 keys
    qd = _t(g["decode_q"])[None, None]
    wd = _t(g["decode_w"])[None, None]
    idx = torch.tensor(out["idx"], dtype=torch.int32)
    cnt = torch.tensor(out["count"], dtype=torch.int32)
    tk = oracle.lightning_topk(qd, wd, K[0], None, idx, cnt, offs, 6)
    assert tk["idx"][0].tolist() == g["topk6_idx"]
    want = [v if v is not None else -math.inf for v in g["topk6_score"]]
    assert tk["score"][0].tolist() == want


def pin_single_head_reduces_to_dot():
    """n_h = 1: x = w * max(0, q . K), a library dot product; w > 0 fetches everything."""
    rng = np.random.default_rng(5)
    S, d_I = 50, 7
    q = rng.standard_normal((1, 1, 1, d_I))
    K = rng.standard_normal((1, S, d_I))
    for wv in (0.8, -0.6):
        out = oracle.score(_t(q), _t([[[wv]]]), _t(K), None, _offs(S))
        qf = _t(q).double().numpy()[0, 0, 0]
        Kf = _t(K).double().numpy()[0]
        dots = np.array([np.dot(qf, Kf[s]) for s in range(S)])
        want = np.float32(wv).astype(np.float64) * np.maximum(dots, 0.0)
        np.testing.assert_allclose(out["x"][0], want, rtol=1e-14, atol=1e-14)
        if wv > 0:
            assert out["mask"].all()
        else:
            assert np.array_equal(out["mask"], (dots <= 0).astype(np.uint8))


def pin_one_hot_keys_pick_a_column():
    """K_s = a e_j: x = sum_h w_h max(0, a q_h[j]) -- catches q stored/indexed transposed."""
    rng = np.random.default_rng(6)
    n_h, d_I = 3, 5
    q = np.round(rng.standard_normal((1, 1, n_h, d_I)) * 4)
    w = np.round(rng.standard_normal((1, 1, n_h)) * 4)
    K = np.zeros((1, 2 * d_I, d_I))
    for j in range(d_I):
        K[0, j, j] = 2.0
        K[0, d_I + j, j] = -1.0
    x = oracle.score(_t(q), _t(w), _t(K), None, _offs(2 * d_I))["x"][0]
    for j in range(d_I):
        assert x[j] == sum(w[0, 0, h] * max(0.0, 2.0 * q[0, 0, h, j]) for h in range(n_h))
        assert x[d_I + j] == sum(w[0, 0, h] * max(0.0, -q[0, 0, h, j]) for h in range(n_h))


def pin_zero_weights_fetch_everything():
    rng = np.random.default_rng(7)
    out = oracle.score(_t(rng.standard_normal((1, 1, 4, 8))), _t(np.zeros((1, 1, 4))),
                       _t(rng.standard_normal((1, 30, 8))), None, _offs(30))
    assert (out["x"] == 0).all() and out["mask"].all() and (out["I"] == 0.5).all()


def pin_homogeneity_and_symmetry():
    """x is linear in w (negating w negates x), positively homogeneous in q and in the key
    scale, invariant to permuting heads, and equivariant to permuting entries."""
    rng = np.random.default_rng(8)
    L, B, n_h, d_I, S = 1, 1, 4, 6, 40
    q = _t(rng.standard_normal((L, B, n_h, d_I)))
    w = _t(rng.standard_normal((L, B, n_h)))
    K = _t(rng.standard_normal((L, S, d_I)))
    sc = _t(rng.uniform(0.5, 2.0, (L, S)))
    offs = _offs(S)
    base = oracle.score(q, w, K, sc, offs)["x"]
    np.testing.assert_allclose(oracle.score(q, -w, K, sc, offs)["x"], -base, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(oracle.score(q * 4, w, K, sc, offs)["x"], 4 * base, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(oracle.score(q, w, K, sc * 2, offs)["x"], 2 * base, rtol=1e-13, atol=1e-13)
    perm = rng.permutation(n_h)
    np.testing.assert_allclose(oracle.score(q[:, :, perm], w[:, :, perm], K, sc, offs)["x"], base,
                               rtol=1e-13, atol=1e-13)
    sp = rng.permutation(S)
    np.testing.assert_allclose(oracle.score(q, w, K[:, sp], sc[:, sp], offs)["x"], base[:, sp],
                               rtol=1e-13, atol=1e-13)
    # a head with weight zero changes nothing
    q2 = torch.cat([q, q[:, :, :1] * 3], dim=2)
    w2 = torch.cat([w, torch.zeros((L, B, 1))], dim=2)
    np.testing.assert_allclose(oracle.score(q2, w2, K, sc, offs)["x"], base, rtol=1e-13, atol=1e-13)


def pin_fp8_and_bf16_keys_equal_f32_keys():
    """Keys given as E4M3 codes with power-of-two scales (or as bf16) score exactly like the
    same values given as fp32 (decoded by torch) -- pins the decode and the scale."""
    rng = np.random.default_rng(9)
    L, B, n_h, d_I, S = 2, 2, 3, 16, 25
    q = _t(rng.standard_normal((L, B, n_h, d_I)), torch.bfloat16)
    w = _t(rng.standard_normal((L, B, n_h)))
    raw = rng.standard_normal((L, B * S, d_I)) * 100
    codes = torch.from_numpy(np.clip(raw, -448, 448).astype(np.float32)).to(torch.float8_e4m3fn)
    sc = torch.from_numpy((2.0 ** rng.integers(-12, -2, (L, B * S))).astype(np.float32))
    offs = _offs(S, S)
    got = oracle.score(q, w, codes, sc, offs)
    Kf = codes.float() * sc[..., None]
    want = oracle.score(q, w, Kf, None, offs)
    assert np.array_equal(got["x"], want["x"]) and np.array_equal(got["mask"], want["mask"])
    Kb = _t(raw / 64, torch.bfloat16)
    assert np.array_equal(oracle.score(q, w, Kb, None, offs)["x"], oracle.score(q, w, Kb.float(), None, offs)["x"])


def pin_or_threshold_and_compaction_invariants():
    rng = np.random.default_rng(10)
    L, B, n_h, d_I = 3, 3, 4, 8
    S = (37, 64, 5)
    offs = _offs(*S)
    q = _t(rng.standard_normal((L, B, n_h, d_I)))
    w = _t(rng.standard_normal((L, B, n_h)) - 0.3)
    K = _t(rng.standard_normal((L, offs[-1], d_I)))
    full = oracle.score(q, w, K, None, offs)
    per = [oracle.score(q[l:l + 1], w[l:l + 1], K[l:l + 1], None, offs)["mask"] for l in range(L)]
    assert np.array_equal(full["mask"], np.bitwise_or.reduce(per))
    for l in range(L):
        assert (full["mask"] >= per[l]).all()
        assert np.array_equal(per[l], (full["x"][l] >= 0).astype(np.uint8))
    prev = full["mask"]
    for thr in (0.55, 0.7, 0.9, 0.99):
        m = oracle.score(q, w, K, None, offs, thr)["mask"]
        assert (m <= prev).all()
        prev = m
        assert np.array_equal(m, np.bitwise_or.reduce(full["x"] >= math.log(thr / (1 - thr))).astype(np.uint8))
    for b in range(B):
        seg = full["mask"][offs[b]:offs[b + 1]]
        assert full["count"][b] == seg.sum()
        assert full["idx"][offs[b]:offs[b] + full["count"][b]].tolist() == np.nonzero(seg)[0].tolist()


def pin_compaction_exhaustive():
    """All 2^10 fetch patterns of a 10-entry sequence: with n_h = 1, w = -1, q = 1 and
    K_s = -1 (fetch) or +1 (skip), x = -max(0, K_s), so the mask must equal the pattern."""
    S = 10
    pats = np.array(list(itertools.product([0, 1], repeat=S)), dtype=np.uint8)
    B = pats.shape[0]
    K = np.where(pats.reshape(-1, 1) == 1, -1.0, 1.0)[None]
    offs = _offs(*([S] * B))
    out = oracle.score(_t(np.ones((1, B, 1, 1))), _t(-np.ones((1, B, 1))), _t(K), None, offs)
    assert np.array_equal(out["mask"], pats.reshape(-1))
    for b in range(B):
        assert out["count"][b] == pats[b].sum()
        assert out["idx"][offs[b]:offs[b] + out["count"][b]].tolist() == np.nonzero(pats[b])[0].tolist()


def pin_score_entries_match_full():
    rng = np.random.default_rng(11)
    L, B, n_h, d_I = 2, 2, 3, 8
    offs = _offs(20, 13)
    q = _t(rng.standard_normal((L, B, n_h, d_I)))
    w = _t(rng.standard_normal((L, B, n_h)))
    K = _t(rng.standard_normal((L, offs[-1], d_I)))
    full = oracle.score(q, w, K, None, offs)["x"]
    eb = np.array([0, 1, 1, 0]); es = np.array([19, 0, 12, 3])
    got = oracle.score_entries(q, w, K, None, offs, eb, es)
    assert np.array_equal(got, full[:, offs[eb] + es])


# ------------------------------------------------------------------ gather and Top-k

def pin_gather_is_row_indexing():
    rng = np.random.default_rng(12)
    offs = _offs(9, 4, 7)
    T = int(offs[-1])
    pool = torch.from_numpy(rng.integers(0, 256, (T, 48), dtype=np.uint8))
    K = _t(rng.standard_normal((T, 8)), torch.bfloat16)
    sc = _t(rng.uniform(size=T))
    idx = np.full(T, -1, np.int32); cnt = np.zeros(3, np.int32)
    for b, sel in enumerate(([0, 3, 8], [], [1, 2, 6])):
        idx[offs[b]:offs[b] + len(sel)] = sel; cnt[b] = len(sel)
    hkv, hK, hsc = oracle.gather(torch.from_numpy(idx), torch.from_numpy(cnt), offs, pool, K, sc, 8)
    for b in range(3):
        for j in range(cnt[b]):
            src = offs[b] + idx[offs[b] + j]
            assert torch.equal(hkv[offs[b] + j], pool[src])
            assert torch.equal(hK[offs[b] + j].view(torch.int16), K[src].view(torch.int16))
            assert hsc[offs[b] + j] == sc[src]


def pin_topk_is_sorted_restriction_of_full_scores():
    """Top-k over the fetched subset = the first k of (all entries' scores restricted to the
    subset) ordered by numpy lexsort (score desc, entry asc); ties included; padding when
    fewer than k entries are fetched."""
    rng = np.random.default_rng(13)
    B, tau, n_h, d_I = 2, 3, 4, 8
    offs = _offs(40, 11)
    T = int(offs[-1])
    qd = _t(rng.standard_normal((B, tau, n_h, d_I)), torch.bfloat16)
    wd = _t(rng.standard_normal((B, tau, n_h)))
    Kraw = rng.standard_normal((T, d_I))
    Kraw[5] = Kraw[9]; Kraw[7] = Kraw[9]                    # exact ties in sequence 0
    K = _t(Kraw, torch.bfloat16)
    all_idx = np.concatenate([np.arange(40), np.arange(11)]).astype(np.int32)
    all_cnt = np.array([40, 11], np.int32)
    full = oracle.lightning_topk(qd, wd, K, None, torch.from_numpy(all_idx), torch.from_numpy(all_cnt),
                                 offs, 5, want_y=True)
    sub = np.full(T, -1, np.int32)
    s0 = np.array([1, 5, 7, 9, 12, 20, 33, 39], np.int32); s1 = np.array([2, 4, 10], np.int32)
    sub[:8] = s0; sub[40:43] = s1
    cnt = np.array([8, 3], np.int32)
    for k in (5, 8):
        got = oracle.lightning_topk(qd, wd, K, None, torch.from_numpy(sub), torch.from_numpy(cnt), offs, k)
        for n in range(B * tau):
            b = n // tau
            sel = s0 if b == 0 else s1
            ys = full["y"][n, offs[b] + sel]
            order = np.lexsort((sel, -ys))[:k]
            want_i = list(sel[order]) + [-1] * (k - len(order))
            want_s = list(ys[order]) + [-math.inf] * (k - len(order))
            assert got["idx"][n].tolist() == want_i
            assert got["score"][n].tolist() == want_s


def pin_topk_single_head_closed_form():
    rng = np.random.default_rng(14)
    offs = _offs(30)
    qd = rng.standard_normal((1, 1, 1, 6)); wd = np.array([[[1.5]]])
    K = rng.standard_normal((30, 6))
    idx = torch.arange(30, dtype=torch.int32); cnt = torch.tensor([30], dtype=torch.int32)
    out = oracle.lightning_topk(_t(qd), _t(wd), _t(K), None, idx, cnt, offs, 30, want_y=True)
    qf = _t(qd).double().numpy()[0, 0, 0]; Kf = _t(K).double().numpy()
    want = 1.5 * np.maximum(Kf @ qf, 0.0)
    np.testing.assert_allclose(out["y"][0], want, rtol=1e-14, atol=1e-14)


# ------------------------------------------------------------------ golden labels (blog review 4.1)

def _golden_rows(rows, p=0.6, theta=1):
    """One sequence, tokens = rows (list of [Lc][S] logit arrays)."""
    z = np.asarray(rows, dtype=np.float32)            # [tau][Lc][S]
    return oracle.golden_labels(z, [0, z.shape[2]], p=p, theta=theta, want_golden=True)


def pin_golden_dominant_entry_is_the_whole_nucleus():
    row = np.zeros(100, dtype=np.float32)
    row[37] = 10.0          # mass 1 against 99 * e^-10 = 0.0045: far above 0.6 of the total
    out = _golden_rows([[row]])
    assert out["nsize"][0, 0, 0] == 1
    assert np.nonzero(out["label"])[0].tolist() == [37]


def pin_golden_uniform_logits_take_ceil_p_s_smallest_entries():
    # equal probabilities 1/S: the nucleus is the first ceil(0.6 S) entries in index order
    for S, want in ((7, 5), (1000, 600), (12, 8), (3, 2)):
        out = _golden_rows([[np.full(S, 0.25, dtype=np.float32)]])
        assert out["nsize"][0, 0, 0] == want, (S, out["nsize"])
        assert np.nonzero(out["label"])[0].tolist() == list(range(want))


def pin_golden_masses_closed_form():
    # probabilities 0.15, 0.55, 0.30 (in that entry order): p = 0.6 needs 0.55 + 0.30
    row = np.log(np.array([0.15, 0.55, 0.30])).astype(np.float32)
    assert np.nonzero(_golden_rows([[row]], p=0.6)["label"])[0].tolist() == [1, 2]
    assert np.nonzero(_golden_rows([[row]], p=0.5)["label"])[0].tolist() == [1]
    assert np.nonzero(_golden_rows([[row]], p=0.9)["label"])[0].tolist() == [0, 1, 2]


def pin_golden_votes_need_theta_layers():
    S, Lc = 20, 5
    layers = np.zeros((Lc, S), dtype=np.float32)
    layers[0:3, 7] = 12.0   # three layers keep entry 7 alone
    layers[3:5, 9] = 12.0   # two layers keep entry 9 alone
    assert np.nonzero(_golden_rows([layers], theta=3)["label"])[0].tolist() == [7]
    assert np.nonzero(_golden_rows([layers], theta=2)["label"])[0].tolist() == [7, 9]
    assert not _golden_rows([layers], theta=6)["label"].any()


def pin_golden_window_is_the_union_of_tokens():
    S, Lc = 16, 3
    t0 = np.zeros((Lc, S), dtype=np.float32)
    t0[:, 4] = 12.0
    t1 = np.zeros((Lc, S), dtype=np.float32)
    t1[:, 11] = 12.0
    out = _golden_rows([t0, t1], theta=3)
    assert np.nonzero(out["golden"][0])[0].tolist() == [4]
    assert np.nonzero(out["golden"][1])[0].tolist() == [11]
    assert np.nonzero(out["label"])[0].tolist() == [4, 11]


def pin_golden_sequences_are_separate_softmaxes():
    S = (7, 0, 4, 4)
    z = np.zeros((1, 1, sum(S)), dtype=np.float32)
    z[0, 0, 0:7] = 0.5                  # sequence 0: uniform, ceil(4.2) = 5 entries
    z[0, 0, 7 + 2] = 12.0               # sequence 2: entry 2 dominates
    z[0, 0, 11:15] = -3.0               # sequence 3: uniform again, ceil(2.4) = 3 entries
    out = oracle.golden_labels(z, [0, 7, 7, 11, 15], theta=1)
    assert out["nsize"][:, 0, 0].tolist() == [5, 0, 1, 3]
    assert np.nonzero(out["label"])[0].tolist() == [0, 1, 2, 3, 4, 9, 11, 12, 13]


def pin_golden_nucleus_is_minimal_and_monotone():
    rng = np.random.default_rng(3)
    S = 500
    row = (rng.standard_normal(S) * 2.0).astype(np.float32)
    row[rng.choice(S, 12, replace=False)] += 6.0
    e = np.exp(row.astype(np.float64) - row.max())
    sets = {}
    for p in (0.3, 0.6, 0.8):
        kept = np.nonzero(_golden_rows([[row]], p=p)["label"])[0]
        sets[p] = set(kept.tolist())
        mass = e[kept].sum()
        assert mass >= p * e.sum() * (1 - 1e-12)                               # reaches p
        assert mass - e[kept].min() < p * e.sum()                              # nothing to spare
        assert e[kept].min() >= np.delete(e, kept).max(initial=0.0)            # the largest ones
    assert sets[0.3] <= sets[0.6] <= sets[0.8]


# ------------------------------------------------------------------ training step (hyper.ai "Method")

def _ones(*shape):
    return torch.ones(shape, dtype=torch.float64)


def pin_train_loss_at_zero_logit():
    # all keys zero: x = 0, p = 1/2 for every entry; BCE is ln 2, focal (gamma 2, alpha 0.25)
    # is at (1/2)^2 ln 2 with at = 0.25 for positives and 0.75 for negatives
    K = torch.zeros((2, 6, 3), dtype=torch.float64)
    lab = [1, 0, 0, 1, 1, 0]
    h = torch.randn((2, 2, 5), dtype=torch.float64)
    W = (torch.randn((2, 4, 5), dtype=torch.float64), torch.randn((2, 6, 4), dtype=torch.float64),
         torch.randn((2, 2, 5), dtype=torch.float64))
    out = oracle.train_step(h, *W, K, None, lab, [0, 2, 6], 2, 3)
    assert abs(out["loss"] - math.log(2.0)) < 1e-15
    assert not out["g_Wdq"].any() and not out["g_Wiuq"].any() and not out["g_Ww"].any()  # ReLU'(0) = 0
    foc = oracle.train_step(h, *W, K, None, lab, [0, 2, 6], 2, 3, gamma=2.0, alpha=0.25)
    want = np.mean([(0.25 if y else 0.75) * 0.25 * math.log(2.0) for y in lab])
    assert abs(foc["loss"] - want) < 1e-15


def pin_train_identity_chain_closed_form():
    # d = r = n_h = d_I = 1 and every weight 1: c = q = w = h = 1, x_s = ReLU(scale_s K_s), and each
    # of the three gradients is (1/T) sum_s (p_s - y_s) ReLU(scale_s K_s) by the chain rule
    K = torch.tensor([[[0.0], [1.5], [-2.0], [0.7], [3.0]]], dtype=torch.float64)
    ks = torch.tensor([[1.0, 0.5, 2.0, 1.0, 0.25]], dtype=torch.float32)
    lab = [1, 0, 1, 0, 1]
    out = oracle.train_step(_ones(1, 1, 1), _ones(1, 1, 1), _ones(1, 1, 1), _ones(1, 1, 1), K, ks, lab, [0, 5], 1, 1)
    x = np.maximum(0.0, K.numpy().ravel() * ks.numpy().ravel().astype(np.float64))
    p = 1.0 / (1.0 + np.exp(-x))
    y = np.array(lab, dtype=np.float64)
    g = ((p - y) * x).sum() / 5
    for k in ("g_Wdq", "g_Wiuq", "g_Ww"):
        assert abs(out[k].item() - g) < 1e-15, k
    assert abs(out["loss"] - np.mean(-(y * np.log(p) + (1 - y) * np.log1p(-p)))) < 1e-14


def _fd_case(seed):
    g = torch.Generator().manual_seed(seed)
    L, B, d, r, n_h, d_I = 2, 2, 6, 4, 3, 5
    S = (5, 7)
    T = sum(S)
    h = torch.randn((L, B, d), generator=g, dtype=torch.float64)
    W = [torch.randn(sh, generator=g, dtype=torch.float64) * 0.7 for sh in ((L, r, d), (L, n_h * d_I, r), (L, n_h, d))]
    K = torch.randn((L, T, d_I), generator=g, dtype=torch.float64)
    ks = (torch.rand((L, T), generator=g) + 0.5).to(torch.float32)
    lab = (torch.rand(T, generator=g) < 0.4).to(torch.uint8).numpy()
    return h, W, K, ks, lab, [0, S[0], T], n_h, d_I


def pin_train_gradients_match_finite_differences():
    # exact inputs (f64): the loss is smooth away from ReLU kinks; central differences of the
    # oracle's own loss check every gradient formula (a dropped term, a wrong sign or a transposed
    # weight would show), for binary cross-entropy and for the focal loss
    for seed, gamma, alpha in ((1, 0.0, -1.0), (2, 2.0, 0.25)):
        h, W, K, ks, lab, offs, n_h, d_I = _fd_case(seed)
        out = oracle.train_step(h, *W, K, ks, lab, offs, n_h, d_I, gamma=gamma, alpha=alpha)
        rng = np.random.default_rng(seed)
        for wi, key in enumerate(("g_Wdq", "g_Wiuq", "g_Ww")):
            for _ in range(6):
                at = tuple(int(rng.integers(0, n)) for n in W[wi].shape)
                eps = 1e-6
                Wp = [w.clone() for w in W]
                Wm = [w.clone() for w in W]
                Wp[wi][at] += eps
                Wm[wi][at] -= eps
                lp = oracle.train_step(h, *Wp, K, ks, lab, offs, n_h, d_I, gamma=gamma, alpha=alpha)["loss"]
                lm = oracle.train_step(h, *Wm, K, ks, lab, offs, n_h, d_I, gamma=gamma, alpha=alpha)["loss"]
                fd = (lp - lm) / (2 * eps)
                assert abs(fd - out[key][at]) <= 1e-7 + 1e-5 * abs(fd), (key, at, fd, out[key][at])


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# ------------------------------------------------------------------ planted mistakes

MUTANTS = {
    "relu_dropped": ("x += (double)w[w0 + hh] * (dot > 0.0 ? dot : 0.0);", "x += (double)w[w0 + hh] * dot;"),
    "strict_threshold": ("if (x >= t)\n                f = 1;", "if (x > t)\n                f = 1;"),
    "q_transposed": ("dot += elem(q, qdt, q0 + (size_t)hh * d_I + e)", "dot += elem(q, qdt, q0 + (size_t)e * n_h + hh)"),
    "scale_dropped": ("        dot *= scale;\n        x +=", "        x +="),
    "and_instead_of_or": ("        int f = 0;\n", "        int f = 0, nf = 0;\n"),
    "tie_breaks_high": ("return (a->s > b->s) - (a->s < b->s);", "return (a->s < b->s) - (a->s > b->s);"),
    "topk_relu_dropped": ("y += (double)w_dec[w0 + hh] * (dot > 0.0 ? dot : 0.0);", "y += (double)w_dec[w0 + hh] * dot;"),
    "c_not_rounded": ("c[j] = round_to(dt, acc);", "c[j] = acc;"),
    "e4m3_bias_off": ("v = ldexp(8.0 + (double)m, e - 10);", "v = ldexp(8.0 + (double)m, e - 9);"),
    "w_uses_wdq": ("acc += elem(h, dt, hb + i) * elem(W_w, dt,", "acc += elem(h, dt, hb + i) * elem(W_dq, dt,"),
    "golden_strict_mass": ("if (mass >= target) break;", "if (mass > target) break;"),
    "golden_vote_off_by_one": ("const uint8_t g = votes >= theta;", "const uint8_t g = votes > theta;"),
    "golden_last_token_only": ("any |= g;", "any = g;"),
    "golden_tie_high": ("if (a->z < b->z) return 1;\n    return (a->s > b->s) - (a->s < b->s);",
                        "if (a->z < b->z) return 1;\n    return (a->s < b->s) - (a->s > b->s);"),
    "golden_mass_not_exp": ("mass += exp(v[r].z - zmax);", "mass += v[r].z - zmax;"),
    "train_relu_grad_dropped": ("                    if (a[hh] > 0.0) {\n                        dw[", "                    if (1) {\n                        dw["),
    "train_dc_transposed": ("acc += dq[lb * nq + o] * elem(W_iuq, dt, ((size_t)l * nq + o) * r + j);",
                            "acc += dq[lb * nq + o] * elem(W_iuq, dt, ((size_t)l * r + j) * nq + o);"),
    "train_focal_sign": ("* lpt * pt * q1 - pow(q1, gamma) * q1) * (y ? 1.0 : -1.0);", "* lpt * pt * q1 - pow(q1, gamma) * q1) * (y ? -1.0 : 1.0);"),
    "train_loss_not_mean": ("*loss_out = loss / N;", "*loss_out = loss;"),
    "train_scale_dropped_in_dq": ("const double gq = g * w[hh] * scale;", "const double gq = g * w[hh];"),
    "golden_softmax_over_all_sequences": ("const float *row = z + ((size_t)i * Lc + l) * (size_t)T + off;",
                                          "const float *row = z + ((size_t)i * Lc + l) * (size_t)T;"),
}


def _extra_edit(name, src):
    if name == "and_instead_of_or":
        # fetched only when every layer passes
        src = src.replace("if (x >= t)\n                f = 1;", "if (x >= t)\n                nf++;")
        src = src.replace("        fetched[row] = (uint8_t)f;", "        fetched[row] = (uint8_t)(nf == L);")
    return src


@pytest.mark.slow
def test_mutants_are_caught(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    with open(os.path.join(os.path.dirname(oracle.__file__), "lsa_oracle.c")) as f:
        src0 = f.read()
    for name, (old, new) in MUTANTS.items():
        assert old in src0, f"mutant {name}: pattern not found in the oracle source"
        src = _extra_edit(name, src0.replace(old, new, 1))
        c = tmp_path / f"{name}.c"
        so = tmp_path / f"{name}.so"
        c.write_text(src)
        subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                        str(c), "-o", str(so), "-lm"], check=True)
        caught = []
        with oracle.using(str(so)):
            for pin in PINS:
                try:
                    pin()
                except AssertionError:
                    caught.append(pin.__name__)
        assert caught, f"mutant {name} passed every pin"

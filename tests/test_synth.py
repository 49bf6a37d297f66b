"""The seeded input generator: deterministic, and a subset of sequences (or a subset of the input
parts) regenerates bit-identically the same values as the full batch, which the full-size parity
tests and the oracle's bounded samples rely on."""
import torch

import synth


def same(x, y):
    """Bitwise equality (1-byte float types compared as their codes)."""
    if x.dtype.itemsize == 1:
        x, y = x.contiguous().view(torch.uint8), y.contiguous().view(torch.uint8)
    return torch.equal(x, y)


def test_same_seed_same_inputs():
    for base in ("ctx128k_bf16", "ctx1m_fp8_b32"):
        wl = synth.workload(base, B=2, S=(700, 129), fetch=(0.2, 0.1), name="det")
        a, b = synth.make_inputs(wl), synth.make_inputs(wl)
        for name in ("h", "W_dq", "W_iuq", "W_w", "q", "w", "K", "pool", "q_dec", "w_dec"):
            x, y = getattr(a, name), getattr(b, name)
            assert x is not None and same(x, y), (base, name)


def test_subset_of_sequences_is_bit_identical():
    for base, kw in (("ctx128k_bf16", dict(B=3, S=(700, 129, 1000), fetch=(0.2, 0.1, 0.3))),
                     ("ctx1m_fp8_b32", dict(B=3, S=(512, 2048, 300), fetch=(0.135,) * 3))):
        wl = synth.workload(base, name="full", **kw)
        full = synth.make_inputs(wl)
        offs = full.seq_offsets.numpy()
        for seqs in ([1], [0, 2], [2, 1]):
            sub = synth.make_inputs(wl.subset(seqs))
            so = sub.seq_offsets.numpy()
            for j, b in enumerate(seqs):
                # per-sequence tensors: [L][B] leading dims
                assert torch.equal(sub.h[:, j], full.h[:, b])
                assert torch.equal(sub.q[:, j], full.q[:, b]) and torch.equal(sub.w[:, j], full.w[:, b])
                assert torch.equal(sub.q_dec[j], full.q_dec[b]) and torch.equal(sub.w_dec[j], full.w_dec[b])
                # entry-axis tensors: segment b of the concatenation
                assert same(sub.K[:, so[j]:so[j + 1]], full.K[:, offs[b]:offs[b + 1]]), (base, seqs, b)
                if full.k_scale is not None:
                    assert torch.equal(sub.k_scale[:, so[j]:so[j + 1]], full.k_scale[:, offs[b]:offs[b + 1]])
                assert torch.equal(sub.pool[so[j]:so[j + 1]], full.pool[offs[b]:offs[b + 1]])
            # weights are per layer, not per sequence
            assert torch.equal(sub.W_dq, full.W_dq) and torch.equal(sub.W_w, full.W_w)


def test_parts_do_not_change_values():
    wl = synth.workload("ctx128k_bf16", B=2, S=(700, 129), fetch=(0.2, 0.1), name="parts")
    full = synth.make_inputs(wl)
    score_only = synth.make_inputs(wl, parts=("score",))
    assert torch.equal(score_only.K, full.K) and torch.equal(score_only.q, full.q)
    assert torch.equal(score_only.w, full.w)
    proj_only = synth.make_inputs(wl, parts=("proj",))
    assert torch.equal(proj_only.h, full.h) and torch.equal(proj_only.W_iuq, full.W_iuq)


def test_calibrated_fetch_rate_through_the_whole_path():
    """The calibration of the head-weight model (synth/fetch_calibration.json, written by
    tests/calibrate_fetch.py) makes the oracle's whole path fetch the wanted share of the 128K
    workload (13.5 %, blog review section 5 table) and of the tiny one (15 %); the planted entries
    of the 128K workload are fetched far more often than the others."""
    import oracle
    for name, tol in (("ctx128k_bf16", 0.002), ("tiny_fp32", 0.02)):
        wl = synth.workload(name)
        assert synth.model_target(wl, 0) != wl.fetch[0], f"{name}: no calibration entry applies"
        inp = synth.make_inputs(wl, parts=("proj", "score"))
        q, w = oracle.project(inp.h, inp.W_dq, inp.W_iuq, inp.W_w, wl.n_h, wl.d_I)
        r = oracle.score(q, w, inp.K, inp.k_scale, inp.seq_offsets.numpy(), want_x=False)
        rate = r["count"].sum() / wl.total_S
        assert abs(rate - wl.fetch[0]) <= tol, (name, rate)
        if wl.planted > 0:
            m = r["mask"].astype(bool)
            pl = inp.planted.any(0).numpy()
            assert m[pl].mean() > 0.95 and m[~pl].mean() < 0.13

"""Indexer training step (lsa_indexer_train_step) against the oracle: loss and the gradients of
W^DQ, W^IUQ, W^w.

Tolerances from the arithmetic: the GPU accumulates in fp32 (about 2^-24 relative per term, sums
of a few thousand terms); with fp32 weights both sides round c and q to fp32 at the same points,
so gradients agree to a relative L2 error far below 1e-4.  With bf16 weights c and q are rounded to
bf16, and a value whose exact sum lies near a rounding boundary may land one bf16 step (2^-8
relative) apart on the two sides; those few flips move the scores and so the gradients, which
are compared to a relative L2 error of 2e-2 (a wrong term, sign or index gives O(1)).
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_kv_cache_memoryindexer_b200 as mod
    return mod


def fp32_case(seed=1):
    g = torch.Generator().manual_seed(seed)
    L, B, d, r, n_h, d_I = 2, 3, 64, 32, 8, 32
    S = (300, 0, 129)
    T = sum(S)
    h = torch.randn((L, B, d), generator=g)
    W = [torch.randn(sh, generator=g) / np.sqrt(sh[-1]) for sh in ((L, r, d), (L, n_h * d_I, r), (L, n_h, d))]
    K = torch.randn((L, T, d_I), generator=g) / np.sqrt(d_I)
    labels = (torch.rand(T, generator=g) < 0.2).to(torch.uint8)
    offs = torch.tensor(np.concatenate([[0], np.cumsum(S)]), dtype=torch.int64)
    return h, W, K, None, labels, offs, n_h, d_I


def bf16_case(kdt, seed=2):
    wl = synth.workload("ctx128k_bf16" if kdt == "bf16" else "ctx1m_fp8_b32", B=2, S=(2000, 700), fetch=(0.135, 0.135),
                        name="train_" + kdt)
    inp = synth.make_inputs(wl, parts=("proj", "score"))
    g = torch.Generator().manual_seed(seed)
    labels = (torch.rand(wl.total_S, generator=g) < 0.15).to(torch.uint8)
    return inp.h, [inp.W_dq, inp.W_iuq, inp.W_w], inp.K, inp.k_scale, labels, inp.seq_offsets, wl.n_h, wl.d_I


def run(m, case, gamma=0.0, alpha=-1.0):
    h, W, K, ks, labels, offs, n_h, d_I = case
    L, B, d = h.shape
    r = W[0].shape[1]
    dev = lambda t: None if t is None else t.cuda()
    loss = torch.zeros(1, dtype=torch.float64, device="cuda")
    gW = [torch.full(w.shape, float("nan"), dtype=torch.float32, device="cuda") for w in W]
    ws = torch.empty(m.lsa_indexer_train_workspace_size(L, B, K.shape[1], d, r, n_h, d_I, h.dtype), dtype=torch.uint8,
                     device="cuda")
    m.lsa_indexer_train_step(dev(h), dev(W[0]), dev(W[1]), dev(W[2]), dev(K), dev(ks), dev(labels), dev(offs), loss,
                             gW[0], gW[1], gW[2], ws, n_h, d_I, gamma=gamma, alpha=alpha)
    m.lsa_check_device()
    ref = oracle.train_step(h, *W, K, ks, labels.numpy(), offs.numpy(), n_h, d_I, gamma=gamma, alpha=alpha)
    return float(loss.item()), [x.cpu().double().numpy() for x in gW], ref


def rel_l2(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


@pytest.mark.parametrize("gamma,alpha", [(0.0, -1.0), (2.0, 0.25)])
def test_train_step_fp32(m, gamma, alpha):
    loss, gW, ref = run(m, fp32_case(), gamma, alpha)
    assert abs(loss - ref["loss"]) <= 1e-5 * abs(ref["loss"])
    for got, key in zip(gW, ("g_Wdq", "g_Wiuq", "g_Ww")):
        assert np.isfinite(got).all()
        assert rel_l2(got, ref[key]) < 1e-4, (key, rel_l2(got, ref[key]))


@pytest.mark.parametrize("kdt", ["bf16", "fp8"])
def test_train_step_bf16_weights(m, kdt):
    loss, gW, ref = run(m, bf16_case(kdt))
    assert abs(loss - ref["loss"]) <= 1e-3 * abs(ref["loss"])
    for got, key in zip(gW, ("g_Wdq", "g_Wiuq", "g_Ww")):
        assert np.isfinite(got).all()
        assert rel_l2(got, ref[key]) < 2e-2, (key, rel_l2(got, ref[key]))


def test_train_step_rejects_unsupported(m):
    h, W, K, ks, labels, offs, n_h, d_I = fp32_case()
    with pytest.raises(m.LSAError, match="dtypes"):
        run(m, (h.to(torch.bfloat16), [w.to(torch.bfloat16) for w in W], K, ks, labels, offs, n_h, d_I))

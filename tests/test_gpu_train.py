"""Indexer training step (lsa_indexer_train_step) against the oracle: loss and the gradients of
W^DQ, W^IUQ, W^w (hyper.ai summary, "Method": only these three matrices are trained, against frozen
keys, with binary cross-entropy and then a focal loss).

Parity rule: element by element.  On exact inputs (tests/parity.py, exact_train_case: every head
dot product, ReLU gate and logit is exact on both sides) each element of the loss and of the three
gradients must lie within its own bound (train_bounds): the fp32 error of the loss derivative and
of every fp32 sum, counted per element from the magnitudes of that element's terms.  Cases: fp32,
bf16 weights with bf16 keys and with E4M3 keys; binary cross-entropy and the focal loss; ragged
sequences (an empty one, tails inside a 128-entry tile) and sequences spanning several CTAs.

The same step on seeded Gaussian inputs (where c and q round to bf16 and a value whose exact sum
lies near a rounding boundary may land one bf16 step apart on the two sides) is also compared as
a whole: relative L2 error 1e-4 with fp32 weights, 2e-2 with bf16 weights.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import check_train, exact_train_case, train_bounds

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


EXACT_DTYPES = [(torch.float32, torch.float32), (torch.bfloat16, torch.bfloat16), (torch.bfloat16, torch.float8_e4m3fn)]


@pytest.mark.parametrize("dt,kdt", EXACT_DTYPES, ids=["f32", "bf16", "bf16-e4m3"])
@pytest.mark.parametrize("gamma,alpha", [(0.0, -1.0), (2.0, 0.25)], ids=["bce", "focal"])
@pytest.mark.parametrize("S", [(300, 0, 129, 517), (2500, 1, 3100)], ids=["ragged", "multi-cta"])
def test_train_step_elementwise(m, dt, kdt, gamma, alpha, S):
    case = exact_train_case(dt, kdt, S=S)
    bounds = train_bounds(case, gamma, alpha)
    loss, gW, ref = run(m, case, gamma, alpha)
    check_train(loss, gW, ref, bounds, what=f"{dt}/{kdt} gamma={gamma} S={S}")

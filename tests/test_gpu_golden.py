"""Golden labels (lsa_golden_labels) against the oracle: label bytes and nucleus sizes exact.

The logits are float32 and both sides take softmax masses and their sums in double, so only a row
whose cumulative mass lands within rounding of p at the boundary could disagree; none does in these
inputs.  Rows of exactly equal logits (ties at the boundary) exercise the entry-order tie rule.
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


def run(m, z, offs, p=0.6, theta=3):
    tau, Lc, T = z.shape
    B = offs.numel() - 1
    label = torch.full((max(T, 1),), 7, dtype=torch.uint8, device="cuda")
    nsize = torch.full((B, tau, Lc), -1, dtype=torch.int32, device="cuda")
    ws = torch.empty(m.lsa_golden_labels_workspace_size(tau, Lc, T), dtype=torch.uint8, device="cuda")
    m.lsa_golden_labels(z.cuda(), offs.cuda(), label, ws, p=p, theta=theta, nsize_out=nsize)
    m.lsa_check_device()
    return label[:T].cpu().numpy(), nsize.cpu().numpy()


def check(m, z, offs, p=0.6, theta=3):
    label, nsize = run(m, z, offs, p, theta)
    ref = oracle.golden_labels(z, offs.numpy(), p=p, theta=theta)
    assert np.array_equal(nsize, ref["nsize"]), f"nucleus sizes differ in {np.argwhere(nsize != ref['nsize'])[:5]}"
    assert np.array_equal(label, ref["label"]), f"{(label != ref['label']).sum()} labels differ"
    return label, ref


def test_golden_ragged(m):
    z, offs = synth.golden_logits((3000, 0, 5000, 129, 1, 64), tau=8, seed=11)
    label, ref = check(m, z, offs)
    assert 0 < label.sum() < label.size


def test_golden_medium(m):
    z, offs = synth.golden_logits((32768, 20000), tau=16, seed=12)
    label, _ = check(m, z, offs)
    assert 100 < label[:32768].sum() < 2000


@pytest.mark.parametrize("p,theta", [(0.6, 1), (0.6, 21), (0.6, 22), (0.3, 3), (0.95, 3), (1.0, 2)])
def test_golden_parameters(m, p, theta):
    z, offs = synth.golden_logits((4000, 777), tau=4, seed=13)
    check(m, z, offs, p=p, theta=theta)


def test_golden_ties_at_the_boundary(m):
    # rows of equal logits: the nucleus is the first ceil(p S) entries; other rows mix a few
    # leaders with a tied remainder so the boundary falls inside the tie
    S = (1000, 7, 333, 64)
    offs = torch.from_numpy(np.concatenate([[0], np.cumsum(S)]).astype(np.int64))
    tau, Lc = 3, 5
    z = torch.zeros((tau, Lc, sum(S)), dtype=torch.float32)
    z[1, :, :] = -1.5
    z[2, :, :] = 0.0
    z[2, :, 5] = 2.0            # leaders in sequence 0, the rest tied
    z[2, :, 17] = 2.0
    z[2, :, 1000 + 7 + 40] = 1.0
    label, ref = check(m, z, offs, theta=3)
    assert ref["nsize"][0, 0, 0] == 600 and ref["nsize"][1, 0, 0] == 5


def test_golden_random_heavy_ties(m):
    # logits drawn from a handful of values: many exact ties everywhere
    g = torch.Generator().manual_seed(3)
    S = (2048, 513)
    offs = torch.from_numpy(np.concatenate([[0], np.cumsum(S)]).astype(np.int64))
    z = torch.randint(0, 6, (4, 21, sum(S)), generator=g).float() * 0.75
    check(m, z, offs)

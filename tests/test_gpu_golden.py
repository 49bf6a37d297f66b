"""Golden labels (lsa_golden_labels) against the oracle: label bytes and nucleus sizes exact.

The logits are float32.  The oracle takes softmax masses and their sums in double.  The kernel takes
the total mass Z in fp32 exp with an error bound, and the candidates' cumulative masses in double;
when the target's interval p [Z - err, Z + err] holds a crossing it recomputes Z in double.  So only
a row whose cumulative mass lands within double rounding of p Z could disagree; none does in these
inputs.  Rows of exactly equal logits (ties at the boundary) exercise the entry-order tie rule, and
the crossing exactly at p Z the recomputation in double.
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


def candidate_set_fits(row, p, cand=4096, depths=(4.0, 8.0, 12.0, 16.0, 24.0, 40.0)):
    """Whether some set of entries within a depth of the row's maximum logit reaches mass p with at
    most `cand` entries (the kernel then sorts that set; otherwise it takes its radix search)."""
    z = row.astype(np.float64)
    e = np.exp(z - z.max())
    for D in depths:
        inside = (np.float32(row.max()) - row) < D
        if e[inside].sum() >= p * e.sum() and inside.sum() <= cand:
            return True
    return False


@pytest.mark.parametrize("p", [0.6, 0.95])
def test_golden_long_flat_rows_take_the_radix_search(m, p):
    # nuclei of thousands of entries within a narrow band of logits: no candidate set of at most
    # 4096 entries reaches p, so every row of the two long sequences runs the radix search (flat
    # logits, and logits from five values with exact ties); the short sequence stays on the sort
    g = torch.Generator().manual_seed(17)
    S = (20000, 9000, 1500)
    offs = torch.from_numpy(np.concatenate([[0], np.cumsum(S)]).astype(np.int64))
    tau, Lc = 2, 3
    z = torch.rand((tau, Lc, sum(S)), generator=g)
    z[1] = torch.randint(0, 5, (Lc, sum(S)), generator=g).float() * 0.01
    zn = z.numpy()
    for i in range(tau):
        for l in range(Lc):
            for b in range(2):
                assert not candidate_set_fits(zn[i, l, offs[b]:offs[b + 1]], p)
    check(m, z, offs, p=p, theta=2)


def test_golden_each_path(m):
    # sequence 0: the entries within 4 of the maximum hold the nucleus (the fast path's candidates);
    # sequence 1: those within 4 hold too little mass, those within 8 (at most 4096) hold it (the
    # general path's candidate sort); sequence 2: the entries within 4 hold too little mass and the
    # rest is flat (the general path's radix search); sequence 3: all equal, the crossing exactly at
    # p Z (the total mass recomputed in double)
    S = (5000, 9000, 30001, 1000)
    offs = torch.from_numpy(np.concatenate([[0], np.cumsum(S)]).astype(np.int64))
    g = torch.Generator().manual_seed(5)
    z = torch.zeros((2, 2, sum(S)), dtype=torch.float32)
    o = offs.numpy()
    z[:, :, o[0]:o[1]] = torch.randn((2, 2, S[0]), generator=g)
    z[:, :, o[0] + 100:o[0] + 400] += 6.0
    z[:, :, o[1]] = 10.0
    z[:, :, o[1] + 1:o[1] + 3001] = 5.0 + 0.01 * torch.randn((2, 2, 3000), generator=g)
    z[:, :, o[1] + 3001:o[2]] = 0.5
    z[:, :, o[2]] = 10.0
    z[:, :, o[2] + 1:o[3]] = torch.rand((2, 2, S[2] - 1), generator=g) * 0.01
    z[:, :, o[3]:o[4]] = -2.0
    zn = z.numpy()
    row1 = zn[0, 0, o[1]:o[2]]
    e1 = np.exp(row1.astype(np.float64) - row1.max())
    near4 = (row1.max() - row1) < 4
    assert e1[near4].sum() < 0.6 * e1.sum() and candidate_set_fits(row1, 0.6)
    row2 = zn[0, 0, o[2]:o[3]]
    assert not candidate_set_fits(row2, 0.6)
    label, ref = check(m, z, offs, p=0.6, theta=1)
    assert ref["nsize"][3, 0, 0] == 600

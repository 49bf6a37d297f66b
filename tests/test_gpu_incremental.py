"""Incremental window-to-window fetch (lsa_fetch_gather_incremental) against the oracle's plain
gather of the new window: the hot buffer must hold the rows of C_t byte for byte, whatever part of
them came from the previous window's buffer, and exactly |C_t minus C_{t-tau}| rows may cross the
host link when the previous lists are ascending.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

ROW = 1024


@pytest.fixture(scope="module")
def m():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_kv_cache_memoryindexer_b200 as mod
    return mod


def offsets(S):
    o = np.zeros(len(S) + 1, dtype=np.int64)
    o[1:] = np.cumsum(S)
    return o


def content(S_max, seed, row=ROW):
    """Row bytes of entry (b, s): the same in every window (a KV row does not change)."""
    return [np.random.default_rng((seed, b)).integers(0, 256, size=(n, row), dtype=np.uint8) for b, n in
            enumerate(S_max)]


def pool_for(rows, S, m, row=ROW):
    o = offsets(S)
    pool = m.MappedPool(int(o[-1]), row)
    for b, n in enumerate(S):
        if n:
            pool.tensor[o[b]:o[b] + n] = torch.from_numpy(rows[b][:n])
    return pool


def lists_to_arrays(lists, S, fill=-7):
    o = offsets(S)
    idx = np.full(max(int(o[-1]), 1), fill, dtype=np.int32)
    cnt = np.zeros(len(S), dtype=np.int32)
    for b, L in enumerate(lists):
        idx[o[b]:o[b] + len(L)] = L
        cnt[b] = len(L)
    return torch.from_numpy(idx), torch.from_numpy(cnt), torch.from_numpy(o)


def run_case(m, S_prev, S_new, prev_lists, new_lists, seed=0, host_check=None, row=ROW):
    rows = content([max(a, b) for a, b in zip(S_prev, S_new)], seed, row)
    pool_prev, pool_new = pool_for(rows, S_prev, m, row), pool_for(rows, S_new, m, row)
    try:
        pi, pc, po = lists_to_arrays(prev_lists, S_prev)
        ni, nc, no = lists_to_arrays(new_lists, S_new)
        Tp, Tn = int(po[-1]), int(no[-1])
        prev_hot, _, _ = oracle.gather(pi, pc, po.numpy(), pool_prev.tensor[:max(Tp, 1)].clone())
        ref_hot, _, _ = oracle.gather(ni, nc, no.numpy(), pool_new.tensor[:max(Tn, 1)].clone())
        hot = torch.zeros((max(Tn, 1), row), dtype=torch.uint8, device="cuda")
        host_rows = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        ws = torch.empty(m.lsa_fetch_incremental_workspace_size(len(S_new), Tn), dtype=torch.uint8, device="cuda")
        m.lsa_fetch_gather_incremental(ni.cuda(), nc.cuda(), no.cuda(), Tn, pi.cuda(), pc.cuda(), po.cuda(), Tp,
                                       prev_hot.cuda(), pool_new.tensor, hot, ws, host_rows_out=host_rows)
        m.lsa_check_device()
        used = np.zeros(max(Tn, 1), dtype=bool)
        for b, L in enumerate(new_lists):
            used[no[b]:no[b] + len(L)] = True
        used = torch.from_numpy(used)
        got = hot.cpu()
        assert torch.equal(got[used], ref_hot[used])
        assert not got[~used].any(), "a slot past a count was written"
        n_host = int(host_rows.item())
        new_only = sum(len(set(N) - set(P)) for N, P in zip(new_lists, prev_lists))
        if host_check is None:
            assert n_host == new_only
        else:
            assert host_check(n_host, new_only, sum(len(N) for N in new_lists))
        return n_host
    finally:
        pool_prev.free()
        pool_new.free()


def drifted(S_prev, S_new, rate, keep, add, seed):
    rng = np.random.default_rng(seed)
    prev, new = [], []
    for b, (sp, sn) in enumerate(zip(S_prev, S_new)):
        P = np.sort(rng.choice(sp, int(rate * sp), replace=False)) if sp else np.zeros(0, dtype=np.int64)
        kept = P[rng.random(P.size) < keep]
        extra = rng.choice(sn, int(add * sn), replace=False) if sn else np.zeros(0, dtype=np.int64)
        grown = np.arange(sp, sn)[rng.random(sn - sp) < 0.5]
        N = np.unique(np.concatenate([kept, extra, grown]).astype(np.int64))
        prev.append(P.astype(np.int32))
        new.append(N.astype(np.int32))
    return prev, new


S_PREV = (3000, 0, 129, 1, 5000, 700, 40)
S_NEW = (3016, 5, 129, 17, 5016, 701, 40)


def test_incremental_drift_ragged(m):
    prev, new = drifted(S_PREV, S_NEW, rate=0.2, keep=0.85, add=0.05, seed=1)
    n_host = run_case(m, S_PREV, S_NEW, prev, new, seed=2)
    assert 0 < n_host < sum(len(N) for N in new)


def test_incremental_same_window_reads_nothing_from_the_host(m):
    prev, _ = drifted(S_PREV, S_PREV, rate=0.3, keep=1.0, add=0.0, seed=3)
    assert run_case(m, S_PREV, S_PREV, prev, prev, seed=4) == 0


def test_incremental_without_previous_rows_reads_everything(m):
    _, new = drifted(S_PREV, S_NEW, rate=0.2, keep=0.0, add=0.3, seed=5)
    prev = [np.zeros(0, dtype=np.int32) for _ in S_PREV]
    assert run_case(m, S_PREV, S_NEW, prev, new, seed=6) == sum(len(N) for N in new)


def test_incremental_unsorted_previous_list_stays_correct(m):
    prev, new = drifted(S_PREV, S_NEW, rate=0.2, keep=0.9, add=0.02, seed=7)
    prev[4] = prev[4][::-1].copy()   # not ascending: lookups may miss, the rows are fetched instead
    run_case(m, S_PREV, S_NEW, prev, new, seed=8, host_check=lambda n, exact, total: exact <= n <= total)


def test_incremental_full_sequences(m):
    S = (64, 300, 2)
    prev = [np.arange(0, 64, 2, dtype=np.int32), np.arange(300, dtype=np.int32), np.zeros(0, dtype=np.int32)]
    new = [np.arange(64, dtype=np.int32), np.arange(1, 300, 3, dtype=np.int32), np.arange(2, dtype=np.int32)]
    assert run_case(m, S, S, prev, new, seed=9) == 32 + 0 + 2


@pytest.mark.parametrize("row", [48, 2048])
def test_incremental_row_sizes(m, row):
    # 3 chunks of 16 bytes per row (most lanes idle) and the largest row (four chunks per lane),
    # through the device copy and the host-link launch
    prev, new = drifted(S_PREV, S_NEW, rate=0.2, keep=0.85, add=0.05, seed=11)
    n_host = run_case(m, S_PREV, S_NEW, prev, new, seed=12, row=row)
    assert 0 < n_host < sum(len(N) for N in new)

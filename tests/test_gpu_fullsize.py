"""Full-size workloads (500K x 8, 1M x 32 with E4M3 keys, the 64-sequence ragged mix) through one
window of IndexerPath, launched exactly as bench.py launches it, checked against the oracle on
sampled outputs and by properties that hold at any size.

Stage 1: every output of three sampled sequences against the oracle projection.
Stages 2-3: sampled entries (random ones plus the first and last entry of every sequence) scored
by the oracle from the GPU's own queries and head weights; fetch decisions bit-exact outside the
2e-3 band around the threshold.
Stage 4a: for every sequence the index list is strictly ascending, inside the sequence, and as long
as the count.
Stage 4b: sampled fetched slots byte-exact against the cold pool and the key rows.
Stage 5: sampled decode queries against the oracle Top-k over the same fetched set.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import check_project, check_topk_query, keys_as_float, li_tolerance, or_exempt

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

N_SAMPLED_ENTRIES = 20000


@pytest.fixture(scope="module")
def m():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_kv_cache_memoryindexer_b200 as mod
    return mod


def run_window(m, wl):
    """One window as bench.py runs it (IndexerPath.run; no optional score or mask outputs)."""
    T = wl.total_S
    pool = m.MappedPool(T, wl.row_bytes)
    inp = synth.make_inputs(wl, pool_out=pool.tensor)
    d = lambda t: None if t is None else t.cuda()
    h, Wdq, Wiuq, Ww = d(inp.h), d(inp.W_dq), d(inp.W_iuq), d(inp.W_w)
    K, ks, offs, qd, wd = d(inp.K), d(inp.k_scale), d(inp.seq_offsets), d(inp.q_dec), d(inp.w_dec)
    path = m.IndexerPath(wl.L, wl.B, wl.d, wl.r, wl.n_h, wl.d_I, wl.tau, wl.k, T, wl.row_bytes,
                         synth.DTYPES[wl.dtype], synth.DTYPES[wl.kdtype])
    path.run(h, Wdq, Wiuq, Ww, K, ks, offs, pool.tensor, qd, wd, sel_layer=wl.sel_layer, threshold=0.5)
    m.lsa_check_device()
    torch.cuda.synchronize()
    del h, Wdq, Wiuq, Ww, K, ks, qd, wd
    return inp, pool, path


@pytest.fixture(scope="module", params=["ctx500k_bf16_b8", "ctx1m_fp8_b32", "ragged_mix_b64"])
def window(request, m):
    wl = synth.workload(request.param)
    inp, pool, path = run_window(m, wl)
    yield wl, inp, pool, path
    del path
    pool.free()
    torch.cuda.empty_cache()


def test_project_sampled_sequences(window):
    wl, inp, _, path = window
    bs = sorted({0, wl.B // 2, wl.B - 1})
    dt = synth.DTYPES[wl.dtype]
    # the workspace of lsa_project holds c [L][B][r] on return
    c = path.ws_proj[:wl.L * wl.B * wl.r * dt.itemsize].view(dt).view(wl.L, wl.B, wl.r)
    check_project(inp.h[:, bs].contiguous(), inp.W_dq, inp.W_iuq, inp.W_w, wl.n_h, wl.d_I,
                  path.q[:, bs].cpu(), path.w[:, bs].cpu(), c[:, bs].cpu(), what=wl.name)


def gpu_mask(path, wl, offs):
    """Fetch mask rebuilt from the index lists (the bench launch writes no mask)."""
    cnt = path.count.cpu().numpy()
    mask = torch.zeros(wl.total_S, dtype=torch.uint8, device="cuda")
    for b in range(wl.B):
        if cnt[b] > 0:
            seg = path.idx[offs[b]:offs[b] + cnt[b]].long() + int(offs[b])
            mask[seg] = 1
    return mask, cnt


def test_compaction_properties(window):
    wl, inp, _, path = window
    offs = inp.seq_offsets.numpy()
    cnt = path.count.cpu().numpy()
    for b in range(wl.B):
        S = int(offs[b + 1] - offs[b])
        assert 0 <= cnt[b] <= S
        if cnt[b] == 0:
            continue
        seg = path.idx[offs[b]:offs[b] + cnt[b]]
        assert int(seg[0]) >= 0 and int(seg[-1]) < S, f"sequence {b}: index outside the sequence"
        assert bool((seg[1:] > seg[:-1]).all()), f"sequence {b}: index list not strictly ascending"
    rate = cnt.sum() / wl.total_S
    assert 0.005 < rate < 0.6  # the synthetic workloads aim at roughly 1-40 % per sequence


def sampled_entries(wl, offs, n, seed):
    rng = np.random.default_rng(seed)
    S = np.diff(offs)
    nz = np.nonzero(S)[0]
    eb = rng.choice(nz, n, p=S[nz] / S[nz].sum()).astype(np.int32)
    es = (rng.random(n) * S[eb]).astype(np.int64)
    edge_b = np.concatenate([nz, nz]).astype(np.int32)
    edge_s = np.concatenate([np.zeros(nz.size, dtype=np.int64), S[nz] - 1])
    return np.concatenate([eb, edge_b]), np.concatenate([es, edge_s])


def test_select_sampled_entries(window):
    wl, inp, _, path = window
    offs = inp.seq_offsets.numpy()
    eb, es = sampled_entries(wl, offs, N_SAMPLED_ENTRIES, seed=11)
    q, w = path.q.cpu(), path.w.cpu()  # the stage's own inputs
    x = oracle.score_entries(q, w, inp.K, inp.k_scale, offs, eb, es)
    I = 1.0 / (1.0 + np.exp(-x))
    ref = (x >= 0.0).any(axis=0)  # threshold 0.5 on the logit
    mask, _ = gpu_mask(path, wl, offs)
    got = mask[torch.from_numpy(offs[eb] + es).cuda()].cpu().numpy().astype(bool)
    ex = or_exempt(I)
    bad = (got != ref) & ~ex
    assert not bad.any(), f"{bad.sum()} of {eb.size} sampled decisions differ outside the band"
    assert ex.mean() < 0.01


def test_gather_sampled_slots(window):
    wl, inp, pool, path = window
    offs = inp.seq_offsets.numpy()
    cnt = path.count.cpu().numpy()
    rng = np.random.default_rng(12)
    bs = np.nonzero(cnt)[0]
    sel = wl.sel_layer
    for b in rng.choice(bs, min(8, bs.size), replace=False):
        js = np.unique(np.concatenate([[0, cnt[b] - 1], rng.integers(0, cnt[b], 256)]))
        slots = torch.from_numpy(offs[b] + js)
        s = path.idx[slots.cuda()].long().cpu()
        rows = offs[b] + s
        assert torch.equal(path.hot_kv[slots.cuda()].cpu(), pool.tensor[rows])
        if inp.k_scale is not None:
            dec = torch.from_numpy(oracle.e4m3_decode(inp.K[sel].view(torch.uint8)[rows].numpy())).float()
            assert torch.equal(path.hot_K[slots.cuda()].cpu().float(), dec)
            assert torch.equal(path.hot_scale[slots.cuda()].cpu(), inp.k_scale[sel][rows])
        else:
            assert torch.equal(path.hot_K[slots.cuda()].cpu(), inp.K[sel][rows])


def test_topk_sampled_queries(window):
    wl, inp, _, path = window
    offs = inp.seq_offsets.numpy()
    idx, cnt = path.idx.cpu(), path.count.cpu()
    rng = np.random.default_rng(13)
    bs = [int(b) for b in rng.choice(np.nonzero(cnt.numpy())[0], 2, replace=False)]
    queries = [(b, int(i)) for b in bs for i in rng.choice(wl.tau, 2, replace=False)]
    sel = wl.sel_layer
    ks = inp.k_scale[sel] if inp.k_scale is not None else None
    ref = oracle.lightning_topk(inp.q_dec, inp.w_dec, inp.K[sel], ks, idx, cnt, offs, wl.k, queries=queries,
                                want_y=True)
    ti, ts = path.topk_idx.cpu().numpy(), path.topk_score.cpu().numpy()
    for n, (b, i) in enumerate(queries):
        F = int(cnt[b])
        s_list = idx[offs[b]:offs[b] + F].numpy()
        rows = torch.from_numpy(offs[b] + s_list.astype(np.int64))
        Krows = inp.K[sel].view(torch.uint8)[rows].view(inp.K.dtype) if ks is not None else inp.K[sel][rows]
        Kf = keys_as_float(Krows, ks[rows] if ks is not None else None)
        tol = li_tolerance(inp.q_dec[b, i], inp.w_dec[b, i], Kf)
        y = ref["y"][n, offs[b]:offs[b] + F]
        check_topk_query(ti[b, i], ts[b, i], y, s_list, tol, wl.k, what=f"{wl.name} query ({b}, {i})")


def test_decode_step_equals_batched_column(window, m):
    """The per-step call at full size, without window entries: step i's Top-k (indices and scores)
    equals column i of the window's batched call bit for bit (the same products and head sums, the
    same ordering of equal scores).  The small-size tests pin both against the oracle."""
    wl, inp, _, path = window
    T = wl.total_S
    qd, wd, offs = inp.q_dec.cuda(), inp.w_dec.cuda(), inp.seq_offsets.cuda()
    ti = torch.empty((wl.B, wl.k), dtype=torch.int32, device="cuda")
    ts = torch.empty((wl.B, wl.k), dtype=torch.float32, device="cuda")
    ws = torch.empty(m.lsa_lightning_topk_step_workspace_size(wl.B, T, wl.n_h, wl.d_I, 0), dtype=torch.uint8,
                     device="cuda")
    for i in (0, wl.tau - 1):
        m.lsa_lightning_topk_step(qd[:, i], wd[:, i], path.hot_K, path.hot_scale, path.idx, path.count, offs, T,
                                  wl.k, ti, ws, topk_score=ts)
        m.lsa_check_device()
        assert torch.equal(ti, path.topk_idx[:, i]), f"{wl.name} step {i}: indices differ"
        assert torch.equal(ts, path.topk_score[:, i]), f"{wl.name} step {i}: scores differ"


def test_fetch_rates_follow_the_workload(window):
    """The whole path fetches the workload's stated share of the entries: about 13.5 % of each
    batch (blog review, section 5 table), each ragged sequence near its own target (1-40 %), and
    the planted entries (relevant to the queries that stage 1 produces) far more often than the rest."""
    wl, inp, _, path = window
    offs = inp.seq_offsets.numpy()
    mask, cnt = gpu_mask(path, wl, offs)
    S = np.asarray(wl.S, dtype=np.float64)
    per = cnt / S
    achieved = float(cnt.sum() / S.sum())
    tgt = np.asarray(wl.fetch)
    if np.ptp(tgt) == 0:
        assert abs(achieved - tgt[0]) <= 0.005, (wl.name, achieved)
    else:
        assert np.abs(per - tgt).max() <= 0.02, (wl.name, np.abs(per - tgt).max())
        assert np.corrcoef(per, tgt)[0, 1] > 0.99
    if wl.planted > 0:
        pl = inp.planted.any(0).numpy()
        got = mask.cpu().numpy().astype(bool)
        assert got[pl].mean() > 0.95 and got[~pl].mean() < 0.15, (got[pl].mean(), got[~pl].mean())

"""Per-step Lightning Top-k (lsa_lightning_topk_step) against the oracle.

At decode step i each sequence has one query; its candidates are the fetched entries plus the
first win_count[b] entries compressed during the window (numbered S_b + j).  The oracle reference
runs the oracle's own Top-k over sequences extended by those entries: the definition itself.
Also: without window entries the step equals column i of the batched call exactly, and tau steps
recorded in a CUDA graph replay to the same results as the eager calls.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import check_topk_query, keys_as_float, li_tolerance

pytestmark = pytest.mark.gpu

W = 16


@pytest.fixture(scope="module")
def m():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_kv_cache_memoryindexer_b200 as mod
    return mod


@pytest.fixture(params=["default", "simt"])
def kernel_path(request, monkeypatch):
    if request.param == "simt":
        monkeypatch.setenv("LSA_DISABLE_TC", "1")
    return request.param


CASES = {
    "bf16": lambda: synth.workload("ctx128k_bf16", B=3, S=(3000, 700, 4100), fetch=(0.2, 0.3, 0.1), name="step_bf16"),
    "fp8": lambda: synth.workload("ctx1m_fp8_b32", B=2, S=(5000, 2600), name="step_fp8"),
    "fp32": lambda: synth.workload("tiny_fp32"),
    # several 2,048-candidate chunks per query (6,000 + window and 2,400 + window candidates), so the
    # select's per-query steps run after chunk CTAs that finish in any order
    "bf16_long": lambda: synth.workload("ctx128k_bf16", B=2, S=(30000, 12000), fetch=(0.2, 0.3),
                                        name="step_bf16_long"),
}
_cache = {}


def case(name):
    if name not in _cache:
        wl = CASES[name]()
        inp = synth.make_inputs(wl, parts=("score", "dec"))
        sel = wl.sel_layer
        Ks = inp.K[sel].contiguous()
        ks = inp.k_scale[sel].contiguous() if inp.k_scale is not None else None
        idx, cnt = synth.random_fetch_list(wl, 0.2, seed=31)
        _, hK, hs = oracle.gather(idx, cnt, inp.seq_offsets.numpy(), None, Ks, ks, wl.d_I)
        if hs is not None:  # the fetch hands E4M3 keys to stage 5 decoded to bf16 (exact)
            hK = hK.float().to(torch.bfloat16)
        Kf = keys_as_float(Ks, ks)
        hot_dt = torch.float32 if wl.kdtype == "f32" else torch.bfloat16
        g = torch.Generator().manual_seed(5)
        winK = (torch.randn((wl.B, W, wl.d_I), generator=g) * Kf.std()).to(hot_dt)
        _cache[name] = (wl, inp, Ks, ks, idx, cnt, hK, hs, winK)
    return _cache[name]


def win_counts(B, i):
    return torch.tensor([min(W, (i + 3 * b) // 4) for b in range(B)], dtype=torch.int32)


def run_step(m, name, i, wc, k, with_window=True):
    wl, inp, Ks, ks, idx, cnt, hK, hs, winK = case(name)
    T = wl.total_S
    ti = torch.empty((wl.B, k), dtype=torch.int32, device="cuda")
    ts = torch.empty((wl.B, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(m.lsa_lightning_topk_step_workspace_size(wl.B, T, wl.n_h, wl.d_I, W if with_window else 0),
                     dtype=torch.uint8, device="cuda")
    qd, wd = inp.q_dec.cuda(), inp.w_dec.cuda()
    kdt = synth.DTYPES[wl.kdtype]
    m.lsa_lightning_topk_step(qd[:, i], wd[:, i], hK.cuda(), None if hs is None else hs.cuda(), idx.cuda(), cnt.cuda(),
                              inp.seq_offsets.cuda(), T, k, ti, ws,
                              win_K=winK.cuda() if with_window else None,
                              win_count=wc.cuda() if with_window else None, topk_score=ts,
                              kdt=m.lsa.DTYPE_CODE[kdt])
    m.lsa_check_device()
    return ti.cpu().numpy(), ts.cpu().numpy()


def check_against_oracle(name, i, wc, k, ti, ts):
    wl, inp, Ks, ks, idx, cnt, hK, hs, winK = case(name)
    offs = inp.seq_offsets.numpy()
    S = np.diff(offs)
    oe = np.zeros(wl.B + 1, dtype=np.int64)
    oe[1:] = np.cumsum(S + W)
    Text = int(oe[-1])
    # keys of the extended sequences as exact fp32 values, scales apart (1 for window entries)
    K_ext = torch.zeros((Text, wl.d_I), dtype=torch.float32)
    ks_ext = torch.ones(Text, dtype=torch.float32) if ks is not None else None
    idx_ext = torch.full((Text,), -1, dtype=torch.int32)
    cnt_ext = torch.zeros(wl.B, dtype=torch.int32)
    for b in range(wl.B):
        K_ext[oe[b]:oe[b] + S[b]] = Ks[offs[b]:offs[b + 1]].float()
        K_ext[oe[b] + S[b]:oe[b + 1]] = winK[b].float()
        if ks is not None:
            ks_ext[oe[b]:oe[b] + S[b]] = ks[offs[b]:offs[b + 1]]
        F, n = int(cnt[b]), int(wc[b])
        idx_ext[oe[b]:oe[b] + F] = idx[offs[b]:offs[b] + F]
        idx_ext[oe[b] + F:oe[b] + F + n] = torch.arange(S[b], S[b] + n, dtype=torch.int32)
        cnt_ext[b] = F + n
    queries = [(b, i) for b in range(wl.B)]
    ref = oracle.lightning_topk(inp.q_dec, inp.w_dec, K_ext, ks_ext, idx_ext, cnt_ext, oe, k, queries=queries,
                                want_y=True)
    for n, (b, _) in enumerate(queries):
        F = int(cnt_ext[b])
        s_list = idx_ext[oe[b]:oe[b] + F].numpy()
        rows = torch.from_numpy(oe[b] + s_list.astype(np.int64))
        Kf = keys_as_float(K_ext[rows], ks_ext[rows] if ks_ext is not None else None)
        tol = li_tolerance(inp.q_dec[b, i], inp.w_dec[b, i], Kf)
        y = ref["y"][n, oe[b]:oe[b] + F]
        check_topk_query(ti[b], ts[b], y, s_list, tol, k, what=f"{name} step {i} seq {b}")


@pytest.mark.parametrize("name", list(CASES))
def test_step_with_window_entries(m, name, kernel_path):
    wl = case(name)[0]
    k = min(wl.k, 256)
    for i in sorted({0, min(5, wl.tau - 1), wl.tau - 1}):
        wc = win_counts(wl.B, i)
        ti, ts = run_step(m, name, i, wc, k)
        check_against_oracle(name, i, wc, k, ti, ts)


@pytest.mark.parametrize("name", ["bf16", "bf16_long"])
def test_step_without_window_equals_batched_column(m, name):
    wl, inp, Ks, ks, idx, cnt, hK, hs, winK = case(name)
    T, k = wl.total_S, 128
    tk = torch.empty((wl.B, wl.tau, k), dtype=torch.int32, device="cuda")
    tsc = torch.empty((wl.B, wl.tau, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(m.lsa_lightning_topk_workspace_size(wl.B, wl.tau, T, k), dtype=torch.uint8, device="cuda")
    m.lsa_lightning_topk(inp.q_dec.cuda(), inp.w_dec.cuda(), hK.cuda(), None, idx.cuda(), cnt.cuda(),
                         inp.seq_offsets.cuda(), T, k, tk, ws, topk_score=tsc)
    m.lsa_check_device()
    for i in (0, 1, 2, 3, 17, wl.tau - 1):
        ti, ts = run_step(m, name, i, None, k, with_window=False)
        assert np.array_equal(ti, tk[:, i].cpu().numpy())
        assert np.array_equal(ts, tsc[:, i].cpu().numpy())


def test_steps_replay_from_a_cuda_graph(m):
    wl, inp, Ks, ks, idx, cnt, hK, hs, winK = case("fp8")
    T, k, tau = wl.total_S, 256, wl.tau
    dev = lambda t: t.cuda()
    qd, wd, hKd, hsd, idd, cnd, od, wKd = (dev(inp.q_dec), dev(inp.w_dec), dev(hK), dev(hs), dev(idx), dev(cnt),
                                           dev(inp.seq_offsets), dev(winK))
    wcs = torch.stack([win_counts(wl.B, i) for i in range(tau)]).cuda()
    ti = torch.zeros((tau, wl.B, k), dtype=torch.int32, device="cuda")
    ts = torch.zeros((tau, wl.B, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(m.lsa_lightning_topk_step_workspace_size(wl.B, T, wl.n_h, wl.d_I, W), dtype=torch.uint8,
                     device="cuda")

    def steps():
        for i in range(tau):
            m.lsa_lightning_topk_step(qd[:, i], wd[:, i], hKd, hsd, idd, cnd, od, T, k, ti[i], ws, win_K=wKd,
                                      win_count=wcs[i], topk_score=ts[i])
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        steps()                      # eager, also the warm-up before capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    m.lsa_check_device()
    eager_i, eager_s = ti.clone(), ts.clone()
    ti.zero_()
    ts.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        steps()
    g.replay()
    torch.cuda.synchronize()
    m.lsa_check_device()
    assert torch.equal(ti, eager_i) and torch.equal(ts, eager_s)
    check_against_oracle("fp8", tau - 1, wcs[tau - 1].cpu(), k, eager_i[tau - 1].cpu().numpy(),
                         eager_s[tau - 1].cpu().numpy())
    del g

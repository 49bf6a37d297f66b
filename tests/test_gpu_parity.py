"""CUDA path vs the CPU oracle, stage by stage and end to end, on seeded synthetic inputs.

Sizes are chosen so the oracle finishes in seconds while spanning many 128-entry tiles and
ragged tails; the full-size workloads, in the launch configuration of bench.py, are covered in
test_gpu_fullsize.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import check_project, check_select, check_topk_query, keys_as_float, li_tolerance, or_exempt

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_kv_cache_memoryindexer_b200 as mod
    return mod


def dev(t):
    return None if t is None else t.cuda()


def ragged_edges():
    """Five sequences with an empty one, a single entry and ragged tails (bf16, 64 x 128)."""
    return synth.workload("ragged_mix_b64", B=5, S=(1000, 0, 129, 4173, 1),
                          fetch=(0.2, 0.1, 0.3, 0.05, 0.5), name="ragged_edges")


def fp8_one_seq():
    return synth.workload("ctx1m_fp8_b32").subset([0])


CASES = {
    "tiny_fp32": lambda: synth.workload("tiny_fp32"),
    "ctx128k_bf16": lambda: synth.workload("ctx128k_bf16"),
    "ragged_edges": ragged_edges,
    "ctx1m_fp8_seq0": fp8_one_seq,
}

_cache = {}


def inputs(name, parts=("score", "pool", "dec")):
    key = (name, parts)
    if key not in _cache:
        wl = CASES[name]()
        _cache[key] = (wl, synth.make_inputs(wl, parts=parts))
    return _cache[key]


def run_select(m, inp, thr=0.5, q=None, w=None):
    wl = inp.wl
    T = wl.total_S
    offs = dev(inp.seq_offsets)
    mask = torch.empty(T, dtype=torch.uint8, device="cuda")
    scores = torch.empty((wl.L, T), dtype=torch.float32, device="cuda")
    idx = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.B, dtype=torch.int32, device="cuda")
    ws = torch.empty(m.lsa_score_select_workspace_size(wl.L, wl.B, T), dtype=torch.uint8, device="cuda")
    m.lsa_memindex_score_select(dev(inp.q if q is None else q), dev(inp.w if w is None else w), dev(inp.K),
                                dev(inp.k_scale), offs, T, thr, idx, cnt, ws, scores_out=scores, mask_out=mask)
    m.lsa_check_device()
    return mask.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy(), scores.cpu().numpy()


# ------------------------------------------------------------------ stages 2-4a

@pytest.fixture(params=["default", "simt"])
def kernel_path(request, monkeypatch):
    """'default' takes the tensor-core kernel where it applies; 'simt' forces the SIMT kernel."""
    if request.param == "simt":
        monkeypatch.setenv("LSA_DISABLE_TC", "1")
    return request.param


@pytest.fixture(params=["pair", "one_cta"])
def e4m3_path(request, monkeypatch):
    """E4M3 keys: 'pair' takes the CTA-pair score kernel (the default), 'one_cta' the one-CTA one."""
    if request.param == "one_cta":
        monkeypatch.setenv("LSA_SCORE_PAIR", "0")
    return request.param


@pytest.mark.parametrize("name", list(CASES))
def test_select_parity(m, name, kernel_path):
    wl, inp = inputs(name)
    offs = inp.seq_offsets.numpy()
    ref = oracle.score(inp.q, inp.w, inp.K, inp.k_scale, offs)
    mask, idx, cnt, I = run_select(m, inp)
    n_ex, n_flip = check_select(mask, idx, cnt, I, ref, offs, what=name)
    assert n_flip <= max(3, n_ex // 10)
    assert cnt.sum() == ref["count"].sum() or n_flip > 0


def test_select_parity_e4m3_one_cta(m, monkeypatch):
    """The one-CTA E4M3 score kernel (taken for more than 1,024 sequences) against the oracle, and
    bit for bit against the CTA-pair kernel."""
    wl, inp = inputs("ctx1m_fp8_seq0")
    monkeypatch.setenv("LSA_SCORE_PAIR", "0")
    offs = inp.seq_offsets.numpy()
    ref = oracle.score(inp.q, inp.w, inp.K, inp.k_scale, offs)
    mask, idx, cnt, I = run_select(m, inp)
    n_ex, n_flip = check_select(mask, idx, cnt, I, ref, offs, what="ctx1m_fp8_seq0 one-CTA")
    assert n_flip <= max(3, n_ex // 10)
    monkeypatch.delenv("LSA_SCORE_PAIR")
    mask2, idx2, cnt2, I2 = run_select(m, inp)
    assert np.array_equal(mask, mask2) and np.array_equal(cnt, cnt2) and np.array_equal(idx, idx2)
    assert np.array_equal(I, I2)


@pytest.mark.parametrize("thr", [0.3, 0.9])
def test_select_thresholds(m, thr):
    wl, inp = inputs("ragged_edges")
    offs = inp.seq_offsets.numpy()
    ref = oracle.score(inp.q, inp.w, inp.K, inp.k_scale, offs, thr)
    mask, idx, cnt, I = run_select(m, inp, thr)
    check_select(mask, idx, cnt, I, ref, offs, thr, what=f"thr={thr}")


def test_select_all_and_none(m):
    wl, inp = inputs("ragged_edges")
    offs = inp.seq_offsets.numpy()
    mask, idx, cnt, _ = run_select(m, inp, 0.5, w=torch.zeros_like(inp.w))      # x = 0 everywhere
    assert mask.all() and np.array_equal(cnt, np.diff(offs))
    mask, idx, cnt, _ = run_select(m, inp, 0.99, w=-torch.abs(inp.w) - 1)       # x <= 0 < logit(0.99)
    assert not mask.any() and (cnt == 0).all()


# ------------------------------------------------------------------ stage 4b

def gather_and_check(m, wl, inp, idx, cnt, mode):
    """mode 'both': rows and keys in one call; 'split': a keys-only call, then a rows-only call (the
    small launch meant for a second stream).  Slots past each count must stay untouched."""
    offs = inp.seq_offsets.numpy()
    T = wl.total_S
    pool = m.MappedPool(T, wl.row_bytes)
    try:
        pool.tensor.copy_(inp.pool)
        hot_kv = torch.zeros((T, wl.row_bytes), dtype=torch.uint8, device="cuda")
        sel = wl.sel_layer
        Ks = dev(inp.K[sel].contiguous())
        ss = dev(inp.k_scale[sel].contiguous()) if inp.k_scale is not None else None
        hot_K = torch.zeros(Ks.shape, dtype=torch.bfloat16 if ss is not None else Ks.dtype, device="cuda")
        hot_s = torch.zeros_like(ss) if ss is not None else None
        di, dc, do = dev(idx), dev(cnt), dev(inp.seq_offsets)
        if mode == "both":
            m.lsa_fetch_gather(di, dc, do, T, pool.tensor, hot_kv, Ks, ss, hot_K, hot_s)
        else:
            m.lsa_fetch_gather(di, dc, do, T, None, None, Ks, ss, hot_K, hot_s)
            m.lsa_fetch_gather(di, dc, do, T, pool.tensor, hot_kv)
        m.lsa_check_device()
        r_kv, r_K, r_s = oracle.gather(idx, cnt, offs, inp.pool, inp.K[sel], inp.k_scale[sel] if ss is not None else None,
                                       wl.d_I)
        used = np.zeros(T, dtype=bool)
        for b in range(wl.B):
            used[offs[b]:offs[b] + cnt[b]] = True
        used = torch.from_numpy(used)
        hk = hot_kv.cpu()
        assert torch.equal(hk[used], r_kv[used])
        assert not hk[~used].any(), "a slot past a count was written"
        if ss is not None:  # E4M3 codes arrive decoded to bf16 (exact)
            r_K = r_K.float().to(torch.bfloat16)
        assert torch.equal(hot_K.cpu()[used].view(torch.uint8), r_K[used].view(torch.uint8))
        if ss is not None:
            assert torch.equal(hot_s.cpu()[used], r_s[used])
    finally:
        pool.free()


@pytest.mark.parametrize("mode", ["both", "split"])
@pytest.mark.parametrize("name", list(CASES))
def test_gather_parity(m, name, mode):
    wl, inp = inputs(name)
    idx, cnt = synth.random_fetch_list(wl, 0.135, seed=3)
    gather_and_check(m, wl, inp, idx, cnt, mode)


def test_gather_rows_many_ragged_sequences(m):
    """300 sequences (several empty, single entries, ragged tails): the rows-only launch numbers all
    fetched rows in one range, so sequence boundaries fall inside warps."""
    S = tuple(1 if i % 13 == 5 else ((i * 37) % 700 if i % 11 else 0) for i in range(300))
    wl = synth.workload("ragged_mix_b64", B=300, S=S, fetch=(0.2,) * 300, name="many_ragged")
    inp = synth.make_inputs(wl, parts=("score", "pool"))
    for rate, seed in ((0.3, 4), (1.0, 5)):
        idx, cnt = synth.random_fetch_list(wl, rate, seed=seed)
        gather_and_check(m, wl, inp, idx, cnt, "split")


# ------------------------------------------------------------------ stage 5

def run_topk(m, inp, idx, cnt, k, pool_needed=False):
    wl = inp.wl
    T = wl.total_S
    sel = wl.sel_layer
    Ks = dev(inp.K[sel].contiguous())
    ss = dev(inp.k_scale[sel].contiguous()) if inp.k_scale is not None else None
    # the hot keys come from the oracle's gather (a byte copy), so this checks stage 5 alone
    _, hK, hs = oracle.gather(idx, cnt, inp.seq_offsets.numpy(), None, inp.K[sel], inp.k_scale[sel] if ss is not None else None,
                              wl.d_I)
    if hs is not None:  # the decode-step kernel takes E4M3 hot keys decoded to bf16 (exact)
        hK = hK.float().to(torch.bfloat16)
    ti = torch.empty((wl.B, wl.tau, k), dtype=torch.int32, device="cuda")
    ts = torch.empty((wl.B, wl.tau, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(m.lsa_lightning_topk_workspace_size(wl.B, wl.tau, T, k), dtype=torch.uint8, device="cuda")
    m.lsa_lightning_topk(dev(inp.q_dec), dev(inp.w_dec), dev(hK), dev(hs), dev(idx), dev(cnt), dev(inp.seq_offsets),
                         T, k, ti, ws, topk_score=ts)
    m.lsa_check_device()
    return ti.cpu().numpy(), ts.cpu().numpy()


def check_topk(inp, idx, cnt, k, ti, ts, queries):
    wl = inp.wl
    offs = inp.seq_offsets.numpy()
    sel = wl.sel_layer
    ref = oracle.lightning_topk(inp.q_dec, inp.w_dec, inp.K[sel], inp.k_scale[sel] if inp.k_scale is not None else None,
                                idx, cnt, offs, k, queries=queries, want_y=True)
    near = 0
    for n, (b, i) in enumerate(queries):
        F = int(cnt[b])
        s_list = idx[offs[b]:offs[b] + F].numpy()
        y = ref["y"][n, offs[b]:offs[b] + F]
        rows = offs[b] + s_list
        Kf = keys_as_float(inp.K[sel][rows], inp.k_scale[sel][rows] if inp.k_scale is not None else None)
        tol = li_tolerance(inp.q_dec[b, i], inp.w_dec[b, i], Kf)
        near += check_topk_query(ti[b, i], ts[b, i], y, s_list, tol, k, what=f"query ({b},{i})")
    return near


@pytest.mark.parametrize("name,k,rate,nq", [("tiny_fp32", 16, 0.135, None), ("ctx128k_bf16", 512, 0.135, None),
                                            ("ragged_edges", 512, 0.2, None), ("ctx1m_fp8_seq0", 2048, 0.135, 6),
                                            ("ctx128k_bf16", 1, 0.05, 8)])
def test_topk_parity(m, name, k, rate, nq):
    wl, inp = inputs(name)
    idx, cnt = synth.random_fetch_list(wl, rate, seed=5)
    ti, ts = run_topk(m, inp, idx, cnt, k)
    qs = [(b, i) for b in range(wl.B) for i in range(wl.tau)]
    if nq is not None:
        rng = np.random.default_rng(1)
        qs = [qs[j] for j in sorted(rng.choice(len(qs), nq, replace=False))]
    check_topk(inp, idx, cnt, k, ti, ts, qs)
    # padding for short sequences and the empty one
    for b in range(wl.B):
        if cnt[b] < k:
            assert (ti[b, :, cnt[b]:] == -1).all()


def test_topk_ties_prefer_smaller_entry(m):
    """Duplicate keys give exactly equal scores; the smaller entry index must come first."""
    wl, inp0 = inputs("ctx128k_bf16")
    inp = synth.Inputs(wl=wl, seq_offsets=inp0.seq_offsets, K=inp0.K.clone(), k_scale=None,
                       q_dec=inp0.q_dec, w_dec=inp0.w_dec)
    inp.K[0, 100:200] = inp.K[0, 5]          # 100 copies of one key
    idx = torch.arange(wl.total_S, dtype=torch.int32)
    cnt = torch.tensor([300], dtype=torch.int32)
    ti, ts = run_topk(m, inp, idx, cnt, 64)
    check_topk(inp, idx, cnt, 64, ti, ts, [(0, 0), (0, 1)])


# ------------------------------------------------------------------ stage 1 and the whole path

PROJ_CASES = {
    "tiny_fp32": lambda: synth.workload("tiny_fp32"),
    "ctx128k_bf16": lambda: synth.workload("ctx128k_bf16"),
    # batch sizes that are not a multiple of the MMA N step (16) and span several 32-column loads
    "b37": lambda: synth.workload("ctx128k_bf16", B=37, S=(64,) * 37, fetch=(0.1,) * 37, name="proj_b37"),
    "b100_small": lambda: synth.workload("ctx128k_bf16", B=100, S=(64,) * 100, fetch=(0.1,) * 100, d=512, r=256,
                                         name="proj_b100"),
    # one layer: 64 tiles of q on 148 SMs, so q is split along r too (slices summed by k_proj_reduce)
    "l1_q_split": lambda: synth.workload("ctx128k_bf16", L=1, name="proj_l1"),
}


@pytest.mark.parametrize("name", list(PROJ_CASES))
def test_project_parity(m, name, kernel_path):
    wl = PROJ_CASES[name]()
    inp = synth.make_inputs(wl, parts=("proj",))
    q_ref, w_ref = oracle.project(inp.h, inp.W_dq, inp.W_iuq, inp.W_w, wl.n_h, wl.d_I)
    q = torch.empty_like(q_ref, device="cuda")
    w = torch.empty_like(w_ref, device="cuda")
    ws = torch.empty(m.lsa_project_workspace_size(wl.L, wl.B, wl.d, wl.r, wl.n_h, wl.d_I, q_ref.dtype),
                     dtype=torch.uint8, device="cuda")
    m.lsa_project(dev(inp.h), dev(inp.W_dq), dev(inp.W_iuq), dev(inp.W_w), q, w, ws)
    m.lsa_check_device()
    # the workspace holds c [L][B][r] on return
    c = ws[:wl.L * wl.B * wl.r * q_ref.dtype.itemsize].view(q_ref.dtype).view(wl.L, wl.B, wl.r)
    check_project(inp.h, inp.W_dq, inp.W_iuq, inp.W_w, wl.n_h, wl.d_I, q.cpu(), w.cpu(), c.cpu(), what=name)


@pytest.mark.parametrize("name", ["tiny_fp32", "ctx128k_bf16"])
def test_whole_path_parity(m, name):
    """One window through IndexerPath.run against the oracle.  Each stage is checked on its own
    inputs (the GPU's outputs of the stage before); the chain as a whole is checked on the fetch
    decisions: equal to the oracle's own chain except entries near the threshold under either
    set of queries (projection roundings may land one bf16 step apart, which moves a score)."""
    wl = CASES[name]()
    inp = synth.make_inputs(wl)
    offs = inp.seq_offsets.numpy()
    T = wl.total_S
    sel = wl.sel_layer
    ks = inp.k_scale
    q_r, w_r = oracle.project(inp.h, inp.W_dq, inp.W_iuq, inp.W_w, wl.n_h, wl.d_I)
    chain = oracle.score(q_r, w_r, inp.K, ks, offs)
    path = m.IndexerPath(wl.L, wl.B, wl.d, wl.r, wl.n_h, wl.d_I, wl.tau, wl.k, T, wl.row_bytes,
                         synth.DTYPES[wl.dtype], synth.DTYPES[wl.kdtype], with_scores=True, with_mask=True)
    pool = m.MappedPool(T, wl.row_bytes)
    try:
        pool.tensor.copy_(inp.pool)
        path.run(dev(inp.h), dev(inp.W_dq), dev(inp.W_iuq), dev(inp.W_w), dev(inp.K), dev(ks), dev(inp.seq_offsets),
                 pool.tensor, dev(inp.q_dec), dev(inp.w_dec), sel_layer=sel)
        m.lsa_check_device()
        mask, idx, cnt = path.mask.cpu().numpy(), path.idx.cpu().numpy(), path.count.cpu().numpy()
        # stage 1 on its inputs
        c = path.ws_proj[:wl.L * wl.B * wl.r * path.q.element_size()].view(path.q.dtype).view(wl.L, wl.B, wl.r)
        check_project(inp.h, inp.W_dq, inp.W_iuq, inp.W_w, wl.n_h, wl.d_I, path.q.cpu(), path.w.cpu(), c.cpu(),
                      what=name)
        # stages 2-4a on their inputs
        stage = oracle.score(path.q.cpu(), path.w.cpu(), inp.K, ks, offs)
        check_select(mask, idx, cnt, path.scores.cpu().numpy(), stage, offs, what=name)
        # the chain's decisions
        ex = or_exempt(chain["I"]) | or_exempt(stage["I"]) | (chain["mask"] != stage["mask"])
        bad = (mask != chain["mask"]) & ~ex
        assert not bad.any(), f"{name}: {bad.sum()} decisions differ from the oracle chain outside the band"
        assert ex.mean() < 0.05  # the band holds a few entries, not the bulk (tiny: 16 of 512)
        # stage 4b and 5 on their inputs (the GPU's index lists)
        ti_, ci_ = torch.from_numpy(idx), torch.from_numpy(cnt)
        r_kv, _, _ = oracle.gather(ti_, ci_, offs, inp.pool, None, None, wl.d_I)
        used = np.zeros(T, dtype=bool)
        for b in range(wl.B):
            used[offs[b]:offs[b] + cnt[b]] = True
        used = torch.from_numpy(used)
        assert torch.equal(path.hot_kv.cpu()[used], r_kv[used])
        ti, ts = path.topk_idx.cpu().numpy(), path.topk_score.cpu().numpy()
        check_topk(inp, ti_, ci_, wl.k, ti, ts, [(b, i) for b in range(wl.B) for i in range(wl.tau)])
    finally:
        pool.free()


# ------------------------------------------------------------------ device-side checks

def test_device_flags_bad_index_and_count(m):
    wl, inp = inputs("ragged_edges")
    T = wl.total_S
    idx, cnt = synth.random_fetch_list(wl, 0.5, seed=9)
    idx[0] = 5000                      # outside sequence 0 (S = 1000)
    pool = m.MappedPool(T, wl.row_bytes)
    try:
        hot = torch.zeros((T, wl.row_bytes), dtype=torch.uint8, device="cuda")
        m.lsa_fetch_gather(dev(idx), dev(cnt), dev(inp.seq_offsets), T, pool.tensor, hot)
        with pytest.raises(m.LSAError, match="index-out-of-range"):
            m.lsa_check_device()
        cnt2 = cnt.clone()
        cnt2[2] = 10_000                 # above S_2 = 129
        idx2, _ = synth.random_fetch_list(wl, 0.5, seed=9)
        m.lsa_fetch_gather(dev(idx2), dev(cnt2), dev(inp.seq_offsets), T, pool.tensor, hot)
        with pytest.raises(m.LSAError, match="count-out-of-range"):
            m.lsa_check_device()
        m.lsa_check_device()             # cleared
    finally:
        pool.free()


def test_device_flags_bad_scale(m):
    wl, inp = inputs("ctx1m_fp8_seq0")
    ks = inp.k_scale.clone()
    ks[1, 77] = -1.0
    T = wl.total_S
    idx = torch.empty(T, dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.B, dtype=torch.int32, device="cuda")
    ws = torch.empty(m.lsa_score_select_workspace_size(wl.L, wl.B, T), dtype=torch.uint8, device="cuda")
    m.lsa_memindex_score_select(dev(inp.q), dev(inp.w), dev(inp.K), dev(ks), dev(inp.seq_offsets), T, 0.5, idx, cnt, ws)
    with pytest.raises(m.LSAError, match="bad-key-scale"):
        m.lsa_check_device()


def test_unmapped_pool_is_rejected(m):
    wl, inp = inputs("tiny_fp32")
    T = wl.total_S
    idx, cnt = synth.random_fetch_list(wl, 0.5)
    hot = torch.zeros((T, wl.row_bytes), dtype=torch.uint8, device="cuda")
    with pytest.raises(m.LSAError, match="LSA_ERR_INVALID_ARG"):
        m.lsa_fetch_gather(dev(idx), dev(cnt), dev(inp.seq_offsets), T, inp.pool, hot)


# ------------------------------------------------------------------ E4M3 code coverage

def _fp8_case(codes_fn, seed):
    wl = synth.workload("ctx1m_fp8_b32", B=2, S=(3000, 1291), fetch=(0.2, 0.2))
    inp = synth.make_inputs(wl, parts=("score",))
    rng = np.random.default_rng(seed)
    codes = codes_fn(rng, inp.K.shape)
    inp.K = torch.from_numpy(codes).view(torch.float8_e4m3fn)
    return wl, inp


def test_select_e4m3_subnormal_codes(m, e4m3_path):
    """Only subnormal E4M3 codes (exponent field 0) with scale 2^9, so every key value is a small
    integer: a flush of subnormals anywhere on the device path would zero every logit."""
    def codes(rng, shape):
        mag = rng.integers(0, 8, size=shape).astype(np.uint8)          # 0x00..0x07
        sign = (rng.random(shape) < 0.5).astype(np.uint8) << 7
        return mag | sign
    wl, inp = _fp8_case(codes, 21)
    inp.k_scale = torch.full_like(inp.k_scale, 512.0)
    offs = inp.seq_offsets.numpy()
    ref = oracle.score(inp.q, inp.w, inp.K, inp.k_scale, offs)
    assert np.abs(ref["x"]).max() > 1.0
    mask, idx, cnt, I = run_select(m, inp)
    check_select(mask, idx, cnt, I, ref, offs, what="subnormal codes")


def test_select_e4m3_all_codes(m, e4m3_path):
    """Every finite E4M3 code (0x7F and 0xFF are NaN and excluded), uniformly, with random scales."""
    def codes(rng, shape):
        c = rng.integers(0, 254, size=shape).astype(np.uint8)          # 0..253
        return np.where(c >= 0x7F, c + 1, c).astype(np.uint8)           # skip 0x7F; 0xFF never drawn
    wl, inp = _fp8_case(codes, 22)
    inp.k_scale = torch.from_numpy(np.random.default_rng(5).uniform(1e-3, 3e-3, inp.k_scale.shape).astype(np.float32))
    offs = inp.seq_offsets.numpy()
    ref = oracle.score(inp.q, inp.w, inp.K, inp.k_scale, offs)
    mask, idx, cnt, I = run_select(m, inp)
    check_select(mask, idx, cnt, I, ref, offs, what="all codes")


# ------------------------------------------------------------------ stage 4b: row sizes

@pytest.mark.parametrize("mode", ["both", "split"])
@pytest.mark.parametrize("row_bytes", [48, 1040, 2048])
def test_gather_row_sizes(m, row_bytes, mode):
    """Rows of 3 chunks of 16 bytes (most lanes idle), of 65 chunks (one lane in the third round) and
    of 128 chunks, the largest row the fetch takes (four chunks per lane): every variant of the
    rows-only launch and the chunk masks of the combined one, with E4M3 keys decoded alongside."""
    wl = synth.workload("ctx1m_fp8_b32", B=3, S=(3000, 0, 1291), fetch=(0.2, 0.2, 0.2), row_bytes=row_bytes,
                        name=f"rows{row_bytes}")
    inp = synth.make_inputs(wl, parts=("score", "pool"))
    idx, cnt = synth.random_fetch_list(wl, 0.3, seed=8)
    gather_and_check(m, wl, inp, idx, cnt, mode)

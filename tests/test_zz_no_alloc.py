"""The allocation-free score/select entry point (lsa_memindex_score_select_static) against the
workspace entry point on the same inputs.

Collected last on purpose (file name): it must pass after every other test has used the library,
as well as alone in a fresh process.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_kv_cache_memoryindexer_b200 as mod
    return mod


def _case(name):
    if name == "bf16":
        wl = synth.workload("ctx128k_bf16", B=3, S=(40000, 1, 12345), fetch=(0.1, 0.5, 0.3), name="static_bf16")
    else:
        wl = synth.workload("ctx1m_fp8_b32", B=2, S=(70000, 333), name="static_fp8")
    inp = synth.make_inputs(wl, parts=("score",))
    d = lambda t: None if t is None else t.cuda()
    return wl, d(inp.q), d(inp.w), d(inp.K), d(inp.k_scale), d(inp.seq_offsets)


def _outputs(wl):
    T = wl.total_S
    return (torch.full((T,), -7, dtype=torch.int32, device="cuda"), torch.empty(wl.B, dtype=torch.int32, device="cuda"),
            torch.empty(T, dtype=torch.uint8, device="cuda"), torch.empty((wl.L, T), dtype=torch.float32, device="cuda"))


def _with_workspace(m, c):
    wl, q, w, K, ks, offs = c
    idx, cnt, mask, sc = _outputs(wl)
    ws = torch.empty(m.lsa_score_select_workspace_size(wl.L, wl.B, wl.total_S), dtype=torch.uint8, device="cuda")
    m.lsa_memindex_score_select(q, w, K, ks, offs, wl.total_S, 0.5, idx, cnt, ws, scores_out=sc, mask_out=mask)
    m.lsa_check_device()
    return idx, cnt, mask, sc


def _static(m, c):
    wl, q, w, K, ks, offs = c
    idx, cnt, mask, sc = _outputs(wl)
    m.lsa_memindex_score_select_static(q, w, K, ks, offs, wl.total_S, 0.5, idx, cnt, scores_out=sc, mask_out=mask)
    m.lsa_check_device()
    return idx, cnt, mask, sc


def _same(a, b):
    idx_a, cnt_a, mask_a, sc_a = a
    idx_b, cnt_b, mask_b, sc_b = b
    assert torch.equal(cnt_a, cnt_b)
    assert torch.equal(mask_a, mask_b)
    assert torch.equal(idx_a, idx_b)  # slots past the counts keep their -7 fill in both
    # same kernels on the same inputs: the scores agree to the last bit; the tolerance of the
    # parity tests (2e-3 on sigmoid scores) is far looser
    assert torch.allclose(sc_a, sc_b, rtol=0, atol=0)


def test_static_matches_workspace_entry_two_calls_in_a_row(m):
    cases = {k: _case(k) for k in ("bf16", "fp8")}
    for name, c in cases.items():
        ref = _with_workspace(m, c)
        assert int(ref[1].sum()) > 0
        first = _static(m, c)
        second = _static(m, c)
        _same(ref, first)
        _same(ref, second)
    # the scratch keeps whatever the previous call left in it: a call on other shapes in between
    # must not change the next result
    other = cases["fp8"]
    _static(m, other)
    again = _static(m, cases["bf16"])
    _same(_with_workspace(m, cases["bf16"]), again)


def test_static_rejects_sizes_beyond_the_scratch(m):
    from sparse_kv_cache_memoryindexer_b200 import lsa
    L, B, T = 3, 128, 16 << 20
    assert lsa.lsa_score_select_workspace_size(L, B, T) > lsa.STATIC_SCORE_SCRATCH_BYTES
    lib = lsa.library()
    p = 256  # never dereferenced: the size check comes first and nothing is launched
    st = lib.lsa_memindex_score_select_static(p, p, p, None, 1, p, T, L, B, 64, 128, 0.5, None, None, p, p, None)
    assert st == 5  # LSA_ERR_WORKSPACE
    msg = lib.lsa_last_error().decode()
    assert "static scratch" in msg and str(lsa.STATIC_SCORE_SCRATCH_BYTES) in msg


def test_static_calls_allocate_no_device_memory(m):
    # the first call on a device looks up the scratch address and loads the kernels; after it,
    # further calls on both key types leave the device's free memory and torch's allocator as
    # they were (outputs are allocated before the measurement)
    cases = {k: _case(k) for k in ("bf16", "fp8")}
    outs = {k: _outputs(c[0]) for k, c in cases.items()}

    def call(k):
        wl, q, w, K, ks, offs = cases[k]
        idx, cnt, mask, sc = outs[k]
        m.lsa_memindex_score_select_static(q, w, K, ks, offs, wl.total_S, 0.5, idx, cnt, scores_out=sc, mask_out=mask)

    for k in cases:
        call(k)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    for _ in range(3):
        for k in cases:
            call(k)
    torch.cuda.synchronize()
    m.lsa_check_device()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    assert torch.cuda.memory_allocated() == alloc0 and torch.cuda.memory_reserved() == reserved0

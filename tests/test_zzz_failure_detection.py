"""Failure detection without a GPU fault: a bounded wait that nothing completes gives up after its
limit, the host reads the timeout from the device error word, and the context stays usable (the
same wait and flag every pipelined kernel uses)."""
import time

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


def test_bounded_wait_gives_up_and_reports(m):
    m.lsa_check_device()                       # nothing pending
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    m.lsa_selftest_wait_timeout(status)
    with pytest.raises(m.LSAError, match="pipeline-wait-timeout"):
        m.lsa_check_device()
    elapsed = time.perf_counter() - t0
    assert status.tolist() == [0, 1]           # the wait did not complete; the abort flag is set
    assert 1.5 < elapsed < 60, elapsed         # it waited for its limit (2 s), then returned
    m.lsa_check_device()                       # the flag was cleared by the read

    # the context is still usable: a small score/select afterwards matches the oracle's lists
    wl = synth.workload("tiny_fp32")
    inp = synth.make_inputs(wl, parts=("score",))
    T = wl.total_S
    idx = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.B, dtype=torch.int32, device="cuda")
    ws = torch.empty(m.lsa_score_select_workspace_size(wl.L, wl.B, T), dtype=torch.uint8, device="cuda")
    m.lsa_memindex_score_select(inp.q.cuda(), inp.w.cuda(), inp.K.cuda(), None, inp.seq_offsets.cuda(), T, 0.5,
                                idx, cnt, ws)
    m.lsa_check_device()
    ref = oracle.score(inp.q, inp.w, inp.K, None, inp.seq_offsets.numpy())
    got_cnt = cnt.cpu().numpy()
    assert np.array_equal(got_cnt, ref["count"])
    assert np.array_equal(idx.cpu().numpy()[:got_cnt[0]], ref["idx"][:got_cnt[0]])

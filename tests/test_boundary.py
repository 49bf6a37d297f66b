"""The C-ABI library: it loads without a GPU, exports every function include/lsa.h declares,
and rejects bad arguments on the host before touching the device."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "include", "lsa.h")


def declared():
    with open(HDR) as f:
        src = f.read()
    return sorted(set(re.findall(r"^(?:lsa_status|size_t|const char \*|uint64_t)\s*\*?\s*(lsa_\w+)\(", src, re.M)))


def test_header_declares_the_hot_path():
    names = declared()
    for n in ("lsa_project", "lsa_memindex_score_select", "lsa_fetch_gather", "lsa_lightning_topk"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from sparse_kv_cache_memoryindexer_b200 import lsa
    out = subprocess.run(["nm", "-D", "--defined-only", lsa.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(lsa_\w+)$", out, re.M))
    missing = [n for n in declared() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    assert set(lsa.EXPORTS) == set(declared())
    for n in declared():
        assert hasattr(lsa.library(), n)


def test_library_is_built_for_sm100a_only():
    from sparse_kv_cache_memoryindexer_b200 import build
    with open(os.path.join(os.path.dirname(build.LIB), "build.log")) as f:
        log = f.read().splitlines()[0]
    assert "arch=compute_100a,code=sm_100a" in log


def test_host_side_validation_without_gpu():
    from sparse_kv_cache_memoryindexer_b200 import lsa
    lib = lsa.library()
    # null pointers are rejected before any CUDA call
    assert lib.lsa_project(None, None, None, None, 1, 1, 1, 8, 8, 1, 1, None, None, None, 0, None) == 1
    assert b"null pointer" in lib.lsa_last_error()
    assert lib.lsa_memindex_score_select(None, None, None, None, 1, None, 0, 1, 1, 1, 1, 0.5, None, None, None,
                                         None, None, 0, None) == 1
    assert lib.lsa_fetch_gather(None, None, None, 0, 1, None, 1024, None, None, None, 0, 0, None, None, None) == 1
    assert lib.lsa_lightning_topk(None, None, None, None, 1, None, None, None, 0, 1, 1, 1, 1, 1, None, None, None, 0,
                                  None) == 1
    # threshold outside (0, 1), k above the maximum, unsupported dtype
    p = C.c_void_p(256)
    assert lib.lsa_memindex_score_select(p, p, p, None, 1, p, 10, 1, 1, 4, 32, 1.5, None, None, p, p, p, 1 << 20,
                                         None) == 1
    assert lib.lsa_lightning_topk(p, p, p, None, 1, p, p, p, 10, 1, 1, 1, 32, 5000, p, None, p, 1 << 20, None) == 1
    assert lib.lsa_project(p, p, p, p, 2, 1, 1, 8, 8, 1, 1, p, p, p, 1 << 20, None) == 2
    # golden labels: vote counts are held in 8 bit slices (at most 255 layers), entries in 32 bits
    assert lib.lsa_golden_labels(p, p, 1000, 1, 4, 256, 0.6, 3, p, None, p, 1 << 20, None) == 1
    assert b"255 layers" in lib.lsa_last_error()
    assert lib.lsa_golden_labels(p, p, 1 << 31, 1, 4, 21, 0.6, 3, p, None, p, 1 << 40, None) == 1
    assert b"2^31" in lib.lsa_last_error()
    # a workspace that is too small
    assert lib.lsa_memindex_score_select(p, p, p, None, 1, p, 1 << 20, 3, 4, 64, 128, 0.5, None, None, p, p, p, 16,
                                         None) == 5
    assert b"workspace needs" in lib.lsa_last_error()


def test_incremental_fetch_host_validation_without_gpu():
    from sparse_kv_cache_memoryindexer_b200 import lsa
    lib = lsa.library()
    p = C.c_void_p(4096)
    args = dict(idx=p, count=p, offs=p, T=100, B=2, pidx=p, pcount=p, poffs=p, pT=100, phot=p, pool=p, rb=1024,
                hot=p, host_rows=None, ws=p, wsb=1 << 20, st=None)

    def call(**kw):
        a = dict(args, **kw)
        return lib.lsa_fetch_gather_incremental(a["idx"], a["count"], a["offs"], a["T"], a["B"], a["pidx"],
                                                a["pcount"], a["poffs"], a["pT"], a["phot"], a["pool"], a["rb"],
                                                a["hot"], a["host_rows"], a["ws"], a["wsb"], a["st"])
    assert call(prev_dummy=None, pidx=None) == 1 and b"null pointer" in lib.lsa_last_error()
    assert call(rb=1000) == 1                                   # not a multiple of 16
    # the two hot buffers overlap (rows 0..99 of each start 1 KB apart)
    assert call(hot=C.c_void_p(1 << 20), phot=C.c_void_p((1 << 20) + 1024)) == 1
    assert b"overlap" in lib.lsa_last_error()
    # a workspace that is too small
    assert call(hot=C.c_void_p(1 << 30), phot=C.c_void_p(1 << 20), wsb=16) == 5
    assert lsa.lsa_fetch_incremental_workspace_size(2, 100) >= 2 * 100 * 4 + 4


def test_workspace_sizes_cover_their_buffers():
    from sparse_kv_cache_memoryindexer_b200 import lsa
    import torch
    T = 262144 * 32
    assert lsa.lsa_score_select_workspace_size(3, 32, T) >= (T // 128) * 16
    assert lsa.lsa_lightning_topk_workspace_size(32, 64, T, 2048) >= 64 * T * 4
    assert lsa.lsa_project_workspace_size(3, 32, 4096, 2048, 64, 128, torch.bfloat16) >= 3 * 32 * 2048 * 2


def test_binding_rejects_wrong_element_types_before_the_device():
    """A pointer carries no element type: the binding checks the widths the C ABI reads (int32
    indices and counts, int64 offsets, fp32 weights and scales, uint8 labels) on the host, so a
    wrong one is an exception, not a kernel reading past a buffer.  CPU tensors: the checks come
    before the device check."""
    import torch
    from sparse_kv_cache_memoryindexer_b200 import lsa
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32)
    i64 = lambda *s: torch.zeros(s, dtype=torch.int64)
    f32 = lambda *s: torch.zeros(s, dtype=torch.float32)
    bf = lambda *s: torch.zeros(s, dtype=torch.bfloat16)
    u8 = lambda *s: torch.zeros(s, dtype=torch.uint8)
    ws = u8(256)
    with pytest.raises(TypeError, match="idx must be torch.int32"):
        lsa.lsa_fetch_gather(i64(10), i32(2), i64(3), 10, None, None, bf(10, 128), None, bf(10, 128))
    with pytest.raises(TypeError, match="seq_offsets must be torch.int64"):
        lsa.lsa_fetch_gather(i32(10), i32(2), i32(3), 10, None, None, bf(10, 128), None, bf(10, 128))
    with pytest.raises(ValueError, match="B \\+ 1 = 3"):
        lsa.lsa_fetch_gather(i32(10), i32(2), i64(4), 10, None, None, bf(10, 128), None, bf(10, 128))
    with pytest.raises(TypeError, match="hot_K must be torch.bfloat16"):   # E4M3 keys arrive as bf16
        lsa.lsa_fetch_gather(i32(10), i32(2), i64(3), 10, None, None,
                             torch.zeros((10, 128), dtype=torch.float8_e4m3fn), f32(10), f32(10, 128), f32(10))
    with pytest.raises(TypeError, match="w must be torch.float32"):
        lsa.lsa_memindex_score_select(bf(3, 2, 64, 128), bf(3, 2, 64), bf(3, 10, 128), None, i64(3), 10, 0.5,
                                      i32(10), i32(2), ws)
    with pytest.raises(TypeError, match="q must be torch.bfloat16"):
        lsa.lsa_memindex_score_select(f32(3, 2, 64, 128), f32(3, 2, 64), bf(3, 10, 128), None, i64(3), 10, 0.5,
                                      i32(10), i32(2), ws)
    with pytest.raises(TypeError, match="count_out must be torch.int32"):
        lsa.lsa_memindex_score_select_static(bf(3, 2, 64, 128), f32(3, 2, 64), bf(3, 10, 128), None, i64(3), 10, 0.5,
                                             i32(10), i64(2))
    with pytest.raises(TypeError, match="q_dec must be torch.bfloat16"):
        lsa.lsa_lightning_topk(f32(2, 4, 64, 128), f32(2, 4, 64), bf(10, 128), None, i32(10), i32(2), i64(3), 10, 8,
                               i32(2, 4, 8), ws)
    with pytest.raises(TypeError, match="win_K must be torch.bfloat16"):
        lsa.lsa_lightning_topk_step(bf(2, 64, 128), f32(2, 64), bf(10, 128), None, i32(10), i32(2), i64(3), 10, 8,
                                    i32(2, 8), ws, win_K=f32(2, 4, 128), win_count=i32(2))
    with pytest.raises(TypeError, match="z must be torch.float32"):
        lsa.lsa_golden_labels(torch.zeros((2, 3, 10), dtype=torch.float64), i64(3), u8(10), ws)
    with pytest.raises(TypeError, match="labels must be torch.uint8"):
        lsa.lsa_indexer_train_step(bf(3, 2, 64), bf(3, 32, 64), bf(3, 64 * 32, 32), bf(3, 64, 64), bf(3, 10, 32),
                                   None, i32(10), i64(3), torch.zeros(1, dtype=torch.float64), f32(3, 32, 64),
                                   f32(3, 64 * 32, 32), f32(3, 64, 64), ws, 64, 32)
    with pytest.raises(TypeError, match="host_rows_out must be torch.int32"):
        lsa.lsa_fetch_gather_incremental(i32(10), i32(2), i64(3), 10, i32(10), i32(2), i64(3), 10, u8(10, 16),
                                         u8(10, 16), u8(10, 16), ws, host_rows_out=i64(1))
    with pytest.raises(ValueError, match="device tensor expected"):     # right types: the device check follows
        lsa.lsa_fetch_gather(i32(10), i32(2), i64(3), 10, None, None, bf(10, 128), None, bf(10, 128))


def test_binding_rejects_buffers_smaller_than_the_call():
    """Capacities follow from the sizes passed (total_S, B, k): a buffer too small for them is an
    exception on the host, never a kernel writing past its end."""
    import torch
    from sparse_kv_cache_memoryindexer_b200 import lsa
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32)
    i64 = lambda *s: torch.zeros(s, dtype=torch.int64)
    f32 = lambda *s: torch.zeros(s, dtype=torch.float32)
    bf = lambda *s: torch.zeros(s, dtype=torch.bfloat16)
    u8 = lambda *s: torch.zeros(s, dtype=torch.uint8)
    ws = u8(256)
    with pytest.raises(ValueError, match="idx_out holds 9 elements, the call needs 10"):
        lsa.lsa_memindex_score_select(bf(3, 2, 64, 128), f32(3, 2, 64), bf(3, 10, 128), None, i64(3), 10, 0.5,
                                      i32(9), i32(2), ws)
    with pytest.raises(ValueError, match="K holds 10 entries per layer, total_S is 11"):
        lsa.lsa_memindex_score_select(bf(3, 2, 64, 128), f32(3, 2, 64), bf(3, 10, 128), None, i64(3), 11, 0.5,
                                      i32(11), i32(2), ws)
    with pytest.raises(ValueError, match="hot_kv holds 1008 bytes, the call needs 1024"):
        lsa.lsa_fetch_gather(i32(64), i32(2), i64(3), 64, u8(64, 16), u8(63, 16))
    with pytest.raises(ValueError, match="hot_K holds"):
        lsa.lsa_fetch_gather(i32(10), i32(2), i64(3), 10, None, None, bf(10, 128), None, bf(9, 128))
    with pytest.raises(ValueError, match="topk_idx holds"):
        lsa.lsa_lightning_topk(bf(2, 4, 64, 128), f32(2, 4, 64), bf(10, 128), None, i32(10), i32(2), i64(3), 10, 8,
                               i32(2, 4, 7), ws)
    with pytest.raises(ValueError, match="topk_idx holds"):
        lsa.lsa_lightning_topk_step(bf(2, 64, 128), f32(2, 64), bf(10, 128), None, i32(10), i32(2), i64(3), 10, 8,
                                    i32(2, 4), ws)
    with pytest.raises(ValueError, match="label_out holds"):
        lsa.lsa_golden_labels(f32(2, 3, 10), i64(3), u8(9), ws)
    with pytest.raises(ValueError, match="prev_hot_kv holds"):
        lsa.lsa_fetch_gather_incremental(i32(10), i32(2), i64(3), 10, i32(10), i32(2), i64(3), 10, u8(9, 16),
                                         u8(10, 16), u8(10, 16), ws)
    with pytest.raises(ValueError, match="g_Wiuq holds"):
        lsa.lsa_indexer_train_step(bf(3, 2, 64), bf(3, 32, 64), bf(3, 64 * 32, 32), bf(3, 64, 64), bf(3, 10, 32),
                                   None, u8(10), i64(3), torch.zeros(1, dtype=torch.float64), f32(3, 32, 64),
                                   f32(3, 64 * 32, 31), f32(3, 64, 64), ws, 64, 32)


def test_binding_host_checks_pass_well_formed_calls():
    """Well-typed, large enough CPU tensors get through every host-side check of every call and
    stop only at the device check (the C library is not called)."""
    import torch
    from sparse_kv_cache_memoryindexer_b200 import lsa
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32)
    i64 = lambda *s: torch.zeros(s, dtype=torch.int64)
    f32 = lambda *s: torch.zeros(s, dtype=torch.float32)
    bf = lambda *s: torch.zeros(s, dtype=torch.bfloat16)
    u8 = lambda *s: torch.zeros(s, dtype=torch.uint8)
    e4 = lambda *s: torch.zeros(s, dtype=torch.float8_e4m3fn)
    ws = u8(256)
    L, B, T, d, r, nh, dI, tau, k, W = 3, 2, 10, 64, 32, 64, 128, 4, 8, 4
    calls = [
        lambda: lsa.lsa_project(bf(L, B, d), bf(L, r, d), bf(L, nh * dI, r), bf(L, nh, d), bf(L, B, nh, dI),
                                f32(L, B, nh), ws),
        lambda: lsa.lsa_memindex_score_select(bf(L, B, nh, dI), f32(L, B, nh), e4(L, T, dI), f32(L, T), i64(B + 1), T,
                                              0.5, i32(T), i32(B), ws, scores_out=f32(L, T), mask_out=u8(T)),
        lambda: lsa.lsa_memindex_score_select_static(f32(L, B, nh, dI), f32(L, B, nh), f32(L, T, dI), None,
                                                     i64(B + 1), T, 0.5, i32(T), i32(B)),
        lambda: lsa.lsa_fetch_gather(i32(T), i32(B), i64(B + 1), T, u8(T, 64), u8(T, 64), e4(T, dI), f32(T),
                                     bf(T, dI), f32(T)),
        lambda: lsa.lsa_fetch_gather_incremental(i32(T), i32(B), i64(B + 1), T, i32(T), i32(B), i64(B + 1), T,
                                                 u8(T, 64), u8(T, 64), u8(T, 64), ws, host_rows_out=i32(1)),
        lambda: lsa.lsa_lightning_topk(bf(B, tau, nh, dI), f32(B, tau, nh), bf(T, dI), f32(T), i32(T), i32(B),
                                       i64(B + 1), T, k, i32(B, tau, k), ws, topk_score=f32(B, tau, k)),
        lambda: lsa.lsa_lightning_topk_step(bf(B, tau, nh, dI)[:, 1], f32(B, tau, nh)[:, 1], bf(T, dI), f32(T),
                                            i32(T), i32(B), i64(B + 1), T, k, i32(B, k), ws, win_K=bf(B, W, dI),
                                            win_scale=f32(B, W), win_count=i32(B), topk_score=f32(B, k)),
        lambda: lsa.lsa_golden_labels(f32(tau, 5, T), i64(B + 1), u8(T), ws, nsize_out=i32(B, tau, 5)),
        lambda: lsa.lsa_indexer_train_step(bf(L, B, d), bf(L, r, d), bf(L, nh * dI, r), bf(L, nh, d), e4(L, T, dI),
                                           f32(L, T), u8(T), i64(B + 1), torch.zeros(1, dtype=torch.float64),
                                           f32(L, r, d), f32(L, nh * dI, r), f32(L, nh, d), ws, nh, dI),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="device tensor expected"):
            call()
    with pytest.raises(TypeError, match="q_out must be torch.bfloat16"):
        lsa.lsa_project(bf(L, B, d), bf(L, r, d), bf(L, nh * dI, r), bf(L, nh, d), f32(L, B, nh, dI), f32(L, B, nh), ws)


def test_build_from_a_clean_tree(tmp_path):
    """__graft_entry__.build() on the committed sources alone (no liblsa.so or oracle library yet)
    compiles both and imports the package."""
    import shutil
    if shutil.which("nvcc") is None or shutil.which("gcc") is None:
        pytest.skip("nvcc and gcc are needed")
    files = subprocess.run(["git", "ls-files"], cwd=ROOT, capture_output=True, text=True, check=True).stdout.split()
    for f in files:
        dst = tmp_path / f
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy2(os.path.join(ROOT, f), dst)
    assert not (tmp_path / "sparse_kv_cache_memoryindexer_b200" / "liblsa.so").exists()
    r = subprocess.run(["python", "-c", "import __graft_entry__ as g; g.build(); "
                        "import sparse_kv_cache_memoryindexer_b200 as m, oracle; print(m.version(), oracle.threads())"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    assert (tmp_path / "sparse_kv_cache_memoryindexer_b200" / "liblsa.so").exists()
    assert (tmp_path / "oracle" / "liblsa_oracle.so").exists()


def test_header_is_plain_c_and_links(tmp_path):
    """include/lsa.h is a C header (C99, no C++ or CUDA types) and a C program links against the
    library with it."""
    import shutil
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    from sparse_kv_cache_memoryindexer_b200 import lsa
    src = tmp_path / "use.c"
    src.write_text('#include "lsa.h"\n#include <stdio.h>\n'
                   'static lsa_status (*const check)(lsa_stream_t) = lsa_check_device;\n'
                   'int main(void) {\n'
                   '  size_t ws = lsa_score_select_workspace_size(3, 2, 100);\n'
                   '  printf("%s %llu %zu\\n", lsa_version(), (unsigned long long)lsa_launch_count(), ws);\n'
                   '  return check == NULL; }\n')
    libdir = os.path.dirname(lsa.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-L", libdir, "-llsa", "-o", str(tmp_path / "use")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr

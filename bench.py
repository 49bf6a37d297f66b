#!/usr/bin/env python
"""Benchmark of the Lookahead Sparse Attention indexer hot path on B200.

One step = one trigger window over one batch of synthetic sequences: project (stage 1),
index score + threshold + OR + compaction (stages 2-4a), fetch from the mapped host cold
pool (4b), and the Lightning-Indexer Top-k of all tau decode queries (5).  Prints ONE JSON
line (rank 0).  `--impl reference` times the CPU oracle instead, on a bounded sample.

Launch: python bench.py [--gpus 1 --steps K --warmup W]; for N > 1 under torchrun, each rank
runs its own batch (independent sequences: weak scaling, no data-path collective).
"""
import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

DEFAULT_WORKLOAD = "ctx1m_fp8_b32"
METRIC = "compressed entries scored+selected/sec at 1M ctx (whole tau-window path)"
UNIT = "entries/s"


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["lsa", "reference"], default="lsa")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    p.add_argument("--batch", type=int, default=0, help="sequences per GPU (default: the workload's batch)")
    p.add_argument("--threshold", type=float, default=0.5)
    p.add_argument("--e2e-steps", type=int, default=0, help="steps of the end-to-end measurement (default: --steps)")
    p.add_argument("--cpu-sample", type=int, default=0,
                   help="entries of the oracle's bounded sample (default: sized for a few minutes of CPU work)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-incremental", action="store_true", help="skip the incremental-fetch measurement")
    p.add_argument("--no-decode-steps", action="store_true", help="skip the per-step decode measurement")
    p.add_argument("--no-golden", action="store_true", help="skip the golden-label measurement")
    p.add_argument("--no-train", action="store_true", help="skip the training-step measurement")
    p.add_argument("--no-steady", action="store_true", help="skip the steady-state window measurement")
    p.add_argument("--no-fetch-rates", action="store_true", help="skip the fetch rates of the other workloads")
    p.add_argument("--only", choices=["golden", "train", "decode"], default=None,
                   help="run only this self-contained measurement (one GPU) and print its JSON line")
    return p.parse_args()


# ------------------------------------------------------------------------------------ ranks

def dist_env():
    """(rank, world size, local rank) from the launcher's environment (1 process without one)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_workload(name, rank, batch=0):
    """The workload of one rank: same shapes on every rank, its own seed (sequences are independent)."""
    base = synth.workload(name)
    over = {"B": batch} if batch else {}
    return synth.workload(name, seed=base.seed + 7919 * rank, **over)


def max_over_ranks(ms, world, device):
    """The job's time is the slowest rank's (every rank takes part in the same collective)."""
    if world <= 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank, steps, elapsed_ms):
    """Units all ranks processed per second of the (max-over-ranks) elapsed time."""
    return world * units_per_rank * steps / (elapsed_ms * 1e-3)


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained", pk["bf16_tflops"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the score kernel,
# from one ncu capture of a smaller batch of the same workload, per entry and layer: the kernel
# streams every key row once, so the traffic grows in proportion to the entries.  Reported only
# while the kernel's sources hash to the value the capture was taken on (null otherwise).
SCORE_TRAFFIC = {
    "fp8": {"bytes_per_entry_layer": 134.11, "capture": "ctx1m_fp8_b32 with B=4 (1,048,576 entries x 3 layers)",
            "kernel": "k_score_pair", "sources": ("score_pair.cuh", "score_tc.cuh", "tc_common.cuh", "common.cuh"),
            "hash": "3a38e0b395165e2e"},
    "bf16": {"bytes_per_entry_layer": 260.23, "capture": "ctx500k_bf16_b8 with B=2 (262,144 entries x 3 layers)",
             "kernel": "k_score_tc<0>", "sources": ("score_tc.cuh", "tc_common.cuh", "common.cuh"),
             "hash": "75fc9bee86641ea6"},
}


def score_kernel_src_hash(sources=("score_tc.cuh", "tc_common.cuh", "common.cuh")):
    import hashlib
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, "sparse_kv_cache_memoryindexer_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def score_traffic(wl):
    tr = SCORE_TRAFFIC.get(wl.kdtype)
    if tr is None or score_kernel_src_hash(tr["sources"]) != tr["hash"]:
        return None, None
    if os.environ.get("LSA_DISABLE_TC"):
        return None, None  # the SIMT kernels run then
    if wl.kdtype == "fp8" and (os.environ.get("LSA_SCORE_PAIR", "1").startswith("0") or wl.B > 1024):
        return None, None  # the one-CTA E4M3 kernel runs then: no capture of its traffic at this version
    return tr["bytes_per_entry_layer"] * wl.L * wl.total_S, tr["kernel"] + ": " + tr["capture"]


# ------------------------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.file = None
        try:
            self.gpu_id = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.gpu_id = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
            if self.gpu_id:
                cmd += ["-i", self.gpu_id]
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.count(",") >= 7]
        os.unlink(self.file.name)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].strip().replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------------ oracle sample

def oracle_sample_workload(wl, n):
    """A bounded sample of the workload: one sequence of n entries, same dims, dtypes and seed."""
    return synth.workload(wl.name, B=1, S=(min(n, wl.S[0]),), fetch=(wl.fetch[0],), seed=wl.seed)


def oracle_step(oracle, wl, inp):
    """The whole path on the CPU oracle for the sample (project, score/OR/compact, gather, Top-k)."""
    offs = inp.seq_offsets.numpy()
    q, w = oracle.project(inp.h, inp.W_dq, inp.W_iuq, inp.W_w, wl.n_h, wl.d_I)
    r = oracle.score(q, w, inp.K, inp.k_scale, offs, want_x=False)
    idx, cnt = torch.from_numpy(r["idx"]), torch.from_numpy(r["count"])
    sel = wl.sel_layer
    ks = inp.k_scale[sel] if inp.k_scale is not None else None
    oracle.gather(idx, cnt, offs, inp.pool, inp.K[sel], ks, wl.d_I)
    oracle.lightning_topk(inp.q_dec, inp.w_dec, inp.K[sel], ks, idx, cnt, offs, wl.k)
    return int(cnt.sum())


def cpu_baseline(wl, n_entries, steps=1):
    import oracle
    sw = oracle_sample_workload(wl, n_entries)
    inp = synth.make_inputs(sw)
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        oracle_step(oracle, sw, inp)
        times.append(time.perf_counter() - t0)
    units = sw.L * sw.total_S
    cores = oracle.threads()
    # the same oracle on one core, over a smaller sample of the same workload
    sw1 = oracle_sample_workload(wl, max(1024, n_entries // 16))
    inp1 = synth.make_inputs(sw1)
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        oracle_step(oracle, sw1, inp1)
        one = sw1.L * sw1.total_S / (time.perf_counter() - t0)
    finally:
        oracle.set_threads(cores)
    return {"value": units / statistics.mean(times), "unit": UNIT, "cores": cores, "kind": "oracle",
            "value_1core": one, "cpu_model": cpu_model(),
            "sample": f"one sequence of {sw.total_S} entries x {sw.L} layers of {wl.name} (same dims/dtypes), "
                      f"whole path incl. S1 projection and Top-k of {sw.tau} queries; mean of {steps} run(s); "
                      f"value_1core: {sw1.total_S} entries on one core"}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# ------------------------------------------------------------------------------------ model of the bytes

def algorithmic(wl, fetched_total):
    """Algorithmic bytes / flops per launch of each stage (the units each launch processes)."""
    T, L, B = wl.total_S, wl.L, wl.B
    eb = {"f32": 4, "bf16": 2, "fp8": 1}
    kb = wl.d_I * eb[wl.kdtype] + (4 if wl.kdtype == "fp8" else 0)       # key bytes per entry per layer
    qb = eb[wl.dtype]
    nq = wl.n_h * wl.d_I
    proj_bytes = L * (wl.r * wl.d + nq * wl.r + wl.n_h * wl.d) * qb + L * B * (wl.d * qb + nq * qb + wl.n_h * 4)
    score_bytes = L * T * kb + L * B * (nq * qb + wl.n_h * 4) + T // 8  # keys + queries and weights + fetch bits
    gather_host = fetched_total * wl.row_bytes                            # crosses the host link
    gather_dev = fetched_total * (wl.row_bytes + wl.d_I * eb[wl.kdtype] * 2 + 8)
    # keys gather: read the key row (+ scale) and the index, write the hot key (bf16 for E4M3) (+ scale)
    kout = wl.d_I * (2 if wl.kdtype == "fp8" else eb[wl.kdtype])
    gather_keys = fetched_total * (wl.d_I * eb[wl.kdtype] + kout + 4 + (8 if wl.kdtype == "fp8" else 0))
    topk_flops = 2.0 * wl.tau * wl.n_h * wl.d_I * fetched_total
    return {"proj_bytes": proj_bytes, "score_bytes": score_bytes, "score_bytes_per_entry_layer": kb,
            "gather_host_bytes": gather_host, "gather_dev_bytes": gather_dev, "gather_key_bytes": gather_keys,
            "topk_flops": topk_flops}


def workload_config(wl, threshold, world):
    """The `config` object of the JSON line: the workload's names and sizes, the same in both arms."""
    alg = algorithmic(wl, 0)
    return {"workload": wl.name, "B": wl.B, "L": wl.L, "S_per_seq": wl.S[0], "d": wl.d, "r": wl.r,
            "n_h": wl.n_h, "d_I": wl.d_I, "tau": wl.tau, "k": wl.k, "kv_row_bytes": wl.row_bytes,
            "keys": wl.kdtype, "threshold": threshold, "parallelism": f"dp{world} (sequences)",
            "l2": "inputs larger than L2 (key stream %.2f GB per step)" % (alg["score_bytes"] / 1e9)}


def h2d_bandwidth(device, nbytes=1 << 30):
    src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(nbytes, dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream(device)
    for _ in range(2):
        dst.copy_(src, non_blocking=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(3):
        dst.copy_(src, non_blocking=True)
    e1.record(st)
    torch.cuda.synchronize(device)
    gbs = 3 * nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del src, dst
    return gbs


# ------------------------------------------------------------------------------------ lsa arm

def measure_train(lsa, device, B=8, S=32768, reps=5):
    """One indexer training step (BCE) on 128K-token shapes: 3 layers, B sequences of S entries,
    d 4096, r 2048, 64 heads x 128, bf16 weights and keys; timed alone.  Roofline: the two per-entry
    products (a = K q^T and dq = G^T K, 4 L T n_h d_I flop) against the sustained bf16 tensor rate."""
    wl = synth.workload("ctx128k_bf16", B=B, S=(S,) * B, fetch=(0.135,) * B, name="train_128k")
    inp = synth.make_inputs(wl, parts=("proj", "score"))
    d = lambda t: t.to(device)
    h, Wdq, Wiuq, Ww, K, offs = d(inp.h), d(inp.W_dq), d(inp.W_iuq), d(inp.W_w), d(inp.K), d(inp.seq_offsets)
    g = torch.Generator().manual_seed(wl.seed + 5)
    labels = d((torch.rand(wl.total_S, generator=g) < 0.135).to(torch.uint8))
    loss = torch.zeros(1, dtype=torch.float64, device=device)
    gW = [torch.empty(w.shape, dtype=torch.float32, device=device) for w in (Wdq, Wiuq, Ww)]
    ws = torch.empty(lsa.lsa_indexer_train_workspace_size(wl.L, B, wl.total_S, wl.d, wl.r, wl.n_h, wl.d_I,
                                                          torch.bfloat16), dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream(device)

    def step():
        lsa.lsa_indexer_train_step(h, Wdq, Wiuq, Ww, K, None, labels, offs, loss, gW[0], gW[1], gW[2], ws, wl.n_h,
                                   wl.d_I, stream=st)
    step()
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(reps):
        step()
    b.record(st)
    torch.cuda.synchronize(device)
    lsa.lsa_check_device(st)
    ms = a.elapsed_time(b) / reps
    flops = 2.0 * 2.0 * wl.L * wl.total_S * wl.n_h * wl.d_I
    peak = load_peaks()["bf16_tflops_sustained"]
    key_bytes = wl.L * wl.total_S * wl.d_I * 2
    out = {"L": wl.L, "B": B, "S": S, "ms": ms, "loss": float(loss.item()),
           "entries_per_s": wl.L * wl.total_S / (ms * 1e-3),
           "roofline": {"bound": "tensor", "achieved": flops / (ms * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                        "peak_note": "sustained bf16 GEMM (measured)",
                        "key_stream_GBps": key_bytes / (ms * 1e-3) / 1e9},
           "note": "forward + BCE + backward of W^DQ, W^IUQ, W^w (projection, per-entry products on tcgen05, "
                   "dc and the three outer products); timed alone"}
    out["roofline"]["frac"] = out["roofline"]["achieved"] / peak
    return out


def measure_golden(lsa, device, B=8, S=32768, tau=64, Lc=21, reps=5):
    """Golden labels of one window for B sequences of S entries (128K-token documents at 4:1),
    tau tokens x Lc CSA layers of raw logits; timed alone.  Roofline: the logits, read once."""
    z, offs = synth.golden_logits([S] * B, tau=tau, Lc=Lc, seed=2024)
    zd, od = z.to(device), offs.to(device)
    T = B * S
    label = torch.empty(T, dtype=torch.uint8, device=device)
    ws = torch.empty(lsa.lsa_golden_labels_workspace_size(tau, Lc, T), dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream(device)
    lsa.lsa_golden_labels(zd, od, label, ws, stream=st)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(reps):
        lsa.lsa_golden_labels(zd, od, label, ws, stream=st)
    b.record(st)
    torch.cuda.synchronize(device)
    lsa.lsa_check_device(st)
    ms = a.elapsed_time(b) / reps
    nbytes = z.numel() * 4 + T
    peaks = load_peaks()
    out = {"B": B, "S": S, "tau": tau, "layers": Lc, "ms": ms, "golden_per_sequence": int(label.sum().item()) / B,
           "roofline": {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "bytes_per_launch": nbytes},
           "note": "softmax + top-p 0.6 + 3-of-21 vote + window union over synthetic logits; timed alone"}
    out["roofline"]["frac"] = out["roofline"]["achieved"] / out["roofline"]["peak"]
    del zd, ws, label
    return out


def measure_decode_steps(lsa, path, wl, offs, qd, wd, st, reps=3):
    """S5 per decode step: tau calls of lsa_lightning_topk_step (one query per sequence each, over
    the fetched entries plus the entries compressed so far in the window: one per 4 steps), eager
    and replayed from a CUDA graph, beside the batched call for all tau queries, each timed alone."""
    tau, B, k, T = wl.tau, wl.B, wl.k, wl.total_S
    W = max(1, tau // 4)
    dev = offs.device
    g = torch.Generator(device="cpu").manual_seed(wl.seed + 23)
    winK = (torch.randn((B, W, wl.d_I), generator=g) * 0.05).to(torch.bfloat16 if wl.kdtype != "f32" else
                                                                   torch.float32).to(dev)
    wcs = torch.tensor([[min(W, i // 4)] * B for i in range(tau)], dtype=torch.int32, device=dev)
    ti = torch.empty((tau, B, k), dtype=torch.int32, device=dev)
    ts = torch.empty((tau, B, k), dtype=torch.float32, device=dev)
    ws = torch.empty(lsa.lsa_lightning_topk_step_workspace_size(B, T, wl.n_h, wl.d_I, W), dtype=torch.uint8, device=dev)

    def steps():
        for i in range(tau):
            lsa.lsa_lightning_topk_step(qd[:, i], wd[:, i], path.hot_K, path.hot_scale, path.idx, path.count, offs, T, k,
                                        ti[i], ws, win_K=winK, win_count=wcs[i], topk_score=ts[i])

    cs = torch.cuda.Stream(device=dev)  # graphs are not captured on the default stream
    cs.wait_stream(st)

    def timed(fn):
        fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(cs)
        for _ in range(reps):
            fn()
        b.record(cs)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    with torch.cuda.stream(cs):
        eager = timed(steps)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cs):
            steps()
        replay = timed(graph.replay)
        batched = timed(lambda: path.topk(qd, wd, offs, cs))
    torch.cuda.synchronize()
    lsa.lsa_check_device(st)
    del graph
    return {"steps": tau, "window_entries_per_sequence": W, "eager_ms_per_step": eager / tau,
            "graph_ms_per_step": replay / tau, "graph_ms_per_window": replay, "batched_ms_per_window": batched,
            "note": "S5 per decode step over the fetched entries plus one new entry per 4 steps; timed alone"}


def measure_decode_only(lsa, device, args):
    """One window of the workload (to fetch the keys), then the per-step decode measurement alone."""
    wl = rank_workload(args.workload, 0, args.batch)
    T = wl.total_S
    pool = lsa.MappedPool(T, wl.row_bytes)
    inp = synth.make_inputs(wl, pool_out=pool.tensor)
    d = lambda t: None if t is None else t.to(device)
    h, Wdq, Wiuq, Ww, K, ks = d(inp.h), d(inp.W_dq), d(inp.W_iuq), d(inp.W_w), d(inp.K), d(inp.k_scale)
    offs, qd, wd = d(inp.seq_offsets), d(inp.q_dec), d(inp.w_dec)
    path = lsa.IndexerPath(wl.L, wl.B, wl.d, wl.r, wl.n_h, wl.d_I, wl.tau, wl.k, T, wl.row_bytes,
                           synth.DTYPES[wl.dtype], synth.DTYPES[wl.kdtype], device=device)
    st = torch.cuda.current_stream(device)
    path.run(h, Wdq, Wiuq, Ww, K, ks, offs, pool.tensor, qd, wd, sel_layer=wl.sel_layer, stream=st)
    torch.cuda.synchronize(device)
    lsa.lsa_check_device(st)
    out = measure_decode_steps(lsa, path, wl, offs, qd, wd, st)
    out["workload"] = wl.name
    pool.free()
    return out


def drifted_lists(idx, cnt, offs, drift, seed):
    """The next window's fetch lists: each sequence keeps 1 - drift of its entries and replaces the
    rest by entries it did not fetch (so the count stays about the same); ascending."""
    rng = np.random.default_rng(seed)
    new_idx = np.full_like(idx, -1)
    new_cnt = np.zeros_like(cnt)
    for b in range(cnt.size):
        S = int(offs[b + 1] - offs[b])
        P = idx[offs[b]:offs[b] + cnt[b]].astype(np.int64)
        kept = P[rng.random(P.size) >= drift]
        free = np.ones(S, dtype=bool)
        free[P] = False
        cand = np.nonzero(free)[0]
        add = rng.choice(cand, min(cand.size, P.size - kept.size), replace=False) if cand.size else cand
        N = np.unique(np.concatenate([kept, add]))
        new_idx[offs[b]:offs[b] + N.size] = N
        new_cnt[b] = N.size
    return new_idx, new_cnt


def measure_incremental(lsa, path, wl, offs, pool, st, drift=0.1, reps=5):
    """S4b incremental: the next window's rows with this window's rows resident (device copies for
    the common entries, the host link for the rest), timed alone on the stream."""
    T = wl.total_S
    offs_h = offs.cpu().numpy()
    idx_n, cnt_n = drifted_lists(path.idx.cpu().numpy(), path.count.cpu().numpy(), offs_h, drift, seed=wl.seed + 17)
    idx_d = torch.from_numpy(idx_n).to(offs.device)
    cnt_d = torch.from_numpy(cnt_n).to(offs.device)
    hot_new = torch.empty_like(path.hot_kv)
    ws = torch.empty(lsa.lsa_fetch_incremental_workspace_size(wl.B, T), dtype=torch.uint8, device=offs.device)
    host_rows = torch.zeros(1, dtype=torch.int32, device=offs.device)

    def call():
        lsa.lsa_fetch_gather_incremental(idx_d, cnt_d, offs, T, path.idx, path.count, offs, T, path.hot_kv,
                                         pool.tensor, hot_new, ws, host_rows_out=host_rows, stream=st)
    for _ in range(2):
        call()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(reps):
        call()
    b.record(st)
    torch.cuda.synchronize()
    lsa.lsa_check_device(st)
    ms = a.elapsed_time(b) / reps
    n_host, rows = int(host_rows.item()), int(cnt_n.sum())
    del hot_new, ws
    return {"drift": drift, "rows": rows, "host_rows": n_host, "ms": ms,
            "host_link_GBps": n_host * wl.row_bytes / (ms * 1e-3) / 1e9,
            "note": "next window = this window with %d %% of each sequence's entries replaced; timed alone"
                    % round(100 * drift)}


def fetched_mask(idx, count, offs):
    """Per-entry fetch decisions [T] (bool, host) from the compacted lists."""
    idx, count, offs = (np.asarray(x) for x in (idx, count, offs))
    m = np.zeros(int(offs[-1]), dtype=bool)
    for b in range(count.size):
        m[offs[b] + idx[offs[b]:offs[b] + count[b]]] = True
    return m


def rate_summary(wl, count, fetched, planted):
    """Achieved fetch rates of one workload against its targets (and of its planted entries)."""
    S = np.asarray(wl.S, dtype=np.float64)
    per = np.asarray(count, dtype=np.float64) / np.maximum(S, 1)
    tgt = np.asarray(wl.fetch, dtype=np.float64)
    out = {"B": wl.B, "target_mean": float((tgt * S).sum() / S.sum()), "achieved": float(per @ S / S.sum())}
    if wl.B > 1:
        dev = per - tgt
        out["per_sequence"] = {"max_abs_dev": float(np.abs(dev).max()), "mean_abs_dev": float(np.abs(dev).mean()),
                               "corr": float(np.corrcoef(per, tgt)[0, 1]) if np.ptp(tgt) > 0 else None}
    if planted is not None and planted.any():
        out["planted_fraction"] = float(planted.mean())
        out["planted_fetched"] = float(fetched[planted].mean())
        out["background_fetched"] = float(fetched[~planted].mean())
    return out


def measure_fetch_rates(lsa, device, skip=()):
    """Whole-path fetch rates (project, score, threshold, OR) of every workload, untimed."""
    out = {}
    for name in synth.WORKLOADS:
        if name in skip:
            continue
        wl = synth.workload(name)
        inp = synth.make_inputs(wl, parts=("proj", "score"))
        d = lambda t: None if t is None else t.to(device)
        dt = synth.DTYPES[wl.dtype]
        q = torch.empty((wl.L, wl.B, wl.n_h, wl.d_I), dtype=dt, device=device)
        w = torch.empty((wl.L, wl.B, wl.n_h), dtype=torch.float32, device=device)
        wsp = torch.empty(max(256, lsa.lsa_project_workspace_size(wl.L, wl.B, wl.d, wl.r, wl.n_h, wl.d_I, dt)),
                          dtype=torch.uint8, device=device)
        lsa.lsa_project(d(inp.h), d(inp.W_dq), d(inp.W_iuq), d(inp.W_w), q, w, wsp)
        T = wl.total_S
        idx = torch.empty(T, dtype=torch.int32, device=device)
        cnt = torch.empty(wl.B, dtype=torch.int32, device=device)
        wss = torch.empty(lsa.lsa_score_select_workspace_size(wl.L, wl.B, T), dtype=torch.uint8, device=device)
        offs = d(inp.seq_offsets)
        lsa.lsa_memindex_score_select(q, w, d(inp.K), d(inp.k_scale), offs, T, 0.5, idx, cnt, wss)
        torch.cuda.synchronize(device)
        lsa.lsa_check_device()
        c = cnt.cpu().numpy()
        m = fetched_mask(idx.cpu().numpy(), c, inp.seq_offsets.numpy())
        out[name] = rate_summary(wl, c, m, inp.planted.any(0).numpy() if wl.planted > 0 else None)
        del q, w, wsp, idx, cnt, wss, offs, inp
    torch.cuda.empty_cache()
    return out


def measure_steady(lsa, path, wl, tensors, pool, st, steps, warmup, drift=0.1):
    """The steady-state window: the same window as the headline step, with the previous window's
    rows resident (its list = this window's with `drift` of each sequence's entries replaced), so
    the rows come from the incremental fetch; timed with the same stage events."""
    h, Wdq, Wiuq, Ww, K, ks, offs, qd, wd, sel = tensors
    T = wl.total_S
    offs_h = offs.cpu().numpy()
    p_idx, p_cnt = drifted_lists(path.idx.cpu().numpy(), path.count.cpu().numpy(), offs_h, drift, seed=wl.seed + 29)
    p_idx, p_cnt = torch.from_numpy(p_idx).to(offs.device), torch.from_numpy(p_cnt).to(offs.device)
    p_hot = torch.empty_like(path.hot_kv)
    lsa.lsa_fetch_gather(p_idx, p_cnt, offs, T, pool.tensor, p_hot, stream=st)   # the previous window's rows
    prev = (p_idx, p_cnt, offs, T, p_hot)

    def window(ev=None):
        path.run(h, Wdq, Wiuq, Ww, K, ks, offs, pool.tensor, qd, wd, sel_layer=sel, stream=st, events=ev, prev=prev)
    for _ in range(warmup):
        window()
    torch.cuda.synchronize()
    evs = []
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
        window(ev)
        evs.append(ev)
    b.record(st)
    torch.cuda.synchronize()
    lsa.lsa_check_device(st)
    ms = a.elapsed_time(b) / steps
    spans = {"project": (0, 1), "score_select": (1, 2), "fetch_keys": (2, 3), "lightning_topk": (3, 4),
             "fetch_rows_incremental (overlapped)": (2, 5), "window": (0, 6)}
    stages = {k: sum(e[i].elapsed_time(e[j]) for e in evs) / steps for k, (i, j) in spans.items()}
    host_rows = int(path.host_rows.item())
    rows = int(path.count.sum().item())
    del p_hot
    return {"window_ms": ms, "entries_per_s": wl.L * T / (ms * 1e-3), "drift": drift, "rows": rows,
            "host_rows": host_rows, "stages_ms": stages, "steps": steps,
            "note": "project + score/select + [rows: incremental fetch from the previous window's hot buffer, "
                    "%d %% of each sequence's entries new | keys + Top-k]; same public call as the headline" % round(100 * drift)}


def run_lsa(args, rank, world, device):
    import sparse_kv_cache_memoryindexer_b200 as lsa
    torch.cuda.set_device(device)
    wl = rank_workload(args.workload, rank, args.batch)
    T = wl.total_S
    dt, kdt = synth.DTYPES[wl.dtype], synth.DTYPES[wl.kdtype]
    pool = lsa.MappedPool(T, wl.row_bytes)
    inp = synth.make_inputs(wl, pool_out=pool.tensor)
    st = torch.cuda.current_stream(device)

    def d(t):
        return None if t is None else t.to(device, non_blocking=False)

    h, Wdq, Wiuq, Ww = d(inp.h), d(inp.W_dq), d(inp.W_iuq), d(inp.W_w)
    K, ks, offs, qd, wd = d(inp.K), d(inp.k_scale), d(inp.seq_offsets), d(inp.q_dec), d(inp.w_dec)
    path = lsa.IndexerPath(wl.L, wl.B, wl.d, wl.r, wl.n_h, wl.d_I, wl.tau, wl.k, T, wl.row_bytes, dt, kdt, device=device,
                           incremental=True)
    sel = wl.sel_layer

    def stages():
        # one window through the public call; events at the stage boundaries of both streams
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
        path.run(h, Wdq, Wiuq, Ww, K, ks, offs, pool.tensor, qd, wd, sel_layer=sel, threshold=args.threshold,
                 stream=st, events=ev)
        return ev

    for _ in range(args.warmup):
        stages()
    torch.cuda.synchronize(device)
    lsa.lsa_check_device(st)
    fetched = int(path.count.sum().item())
    head_rates = rate_summary(wl, path.count.cpu().numpy(),
                              fetched_mask(path.idx.cpu().numpy(), path.count.cpu().numpy(), inp.seq_offsets.numpy()),
                              inp.planted.any(0).numpy() if wl.planted > 0 else None)
    h2d = h2d_bandwidth(device)

    clocks = ClockSampler(device)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    n0 = lsa.launch_count()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(st)
    evs = [stages() for _ in range(args.steps)]
    t1.record(st)
    torch.cuda.synchronize(device)
    launches = lsa.launch_count() - n0
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    lsa.lsa_check_device(st)
    elapsed_ms = t0.elapsed_time(t1)
    # project, select, keys gather, Top-k (main stream); rows gather (second stream, from the end of
    # select); whole window
    spans = ((0, 1), (1, 2), (2, 3), (3, 4), (2, 5), (0, 6))
    stage_ms = np.zeros(len(spans))
    for ev in evs:
        for i, (a, b) in enumerate(spans):
            stage_ms[i] += ev[a].elapsed_time(ev[b])
    stage_ms /= args.steps
    elapsed_ms = max_over_ranks(elapsed_ms, world, device)

    # end to end through the public API with host buffers.  Per window the host supplies the trigger
    # hidden states, the decode queries and weights, and the index keys of the entries compressed
    # during the window (tau/4 per sequence and layer at 4:1, written into the last tau/4 slots of
    # each sequence); the index-key cache itself stays on the device like the weights (the method
    # offloads the compressed KV rows, which the fetch reads from the host pool inside the window).
    e2e = None
    if not args.no_e2e:
        Wn = max(1, wl.tau // 4)
        offs_h = inp.seq_offsets.numpy()
        rows = np.array([l * T + offs_h[b + 1] - Wn + j for l in range(wl.L) for b in range(wl.B)
                         for j in range(Wn) if offs_h[b + 1] - offs_h[b] >= Wn], dtype=np.int64)
        rows_d = torch.from_numpy(rows).to(device)
        kraw = (lambda t: t.view(torch.uint8)) if inp.K.dtype == torch.float8_e4m3fn else (lambda t: t)
        host = {"h": inp.h.pin_memory(), "qd": inp.q_dec.pin_memory(), "wd": inp.w_dec.pin_memory(),
                "K_new": kraw(inp.K).reshape(-1, wl.d_I)[torch.from_numpy(rows)].pin_memory()}
        stage = {"K_new": torch.empty_like(host["K_new"], device=device)}
        if inp.k_scale is not None:
            host["ks_new"] = inp.k_scale.reshape(-1)[torch.from_numpy(rows)].pin_memory()
            stage["ks_new"] = torch.empty_like(host["ks_new"], device=device)
        K_rows = kraw(K).view(-1, wl.d_I)
        out_i = torch.empty(path.topk_idx.shape, dtype=torch.int32).pin_memory()
        out_c = torch.empty(path.count.shape, dtype=torch.int32).pin_memory()
        h2d_b = sum(v.numel() * v.element_size() for v in host.values())
        d2h_b = out_i.numel() * 4 + out_c.numel() * 4

        def e2e_step():
            h.copy_(host["h"], non_blocking=True)
            qd.copy_(host["qd"], non_blocking=True)
            wd.copy_(host["wd"], non_blocking=True)
            stage["K_new"].copy_(host["K_new"], non_blocking=True)
            K_rows.index_copy_(0, rows_d, stage["K_new"])
            if ks is not None:
                stage["ks_new"].copy_(host["ks_new"], non_blocking=True)
                ks.view(-1).index_copy_(0, rows_d, stage["ks_new"])
            path.run(h, Wdq, Wiuq, Ww, K, ks, offs, pool.tensor, qd, wd, sel_layer=sel, threshold=args.threshold,
                     stream=st)
            out_i.copy_(path.topk_idx, non_blocking=True)
            out_c.copy_(path.count, non_blocking=True)

        e2e_steps = args.e2e_steps or args.steps
        e2e_step()
        torch.cuda.synchronize(device)
        if world > 1:
            torch.distributed.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(e2e_steps):
            e2e_step()
        b.record(st)
        torch.cuda.synchronize(device)
        e_ms = a.elapsed_time(b)
        e_ms = max_over_ranks(e_ms, world, device)
        e2e = {"value": job_throughput(world, wl.L * T, e2e_steps, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b,
               "ms_per_step": e_ms / e2e_steps, "steps": e2e_steps,
               "inputs": "per window: trigger hidden states, decode queries and weights, the index keys (and scales) "
                         "of the %d entries per sequence and layer compressed during the window; out: Top-k indices "
                         "and fetched counts" % Wn}
        del host

    steady = None
    if not args.no_steady and world == 1:
        steady = measure_steady(lsa, path, wl, (h, Wdq, Wiuq, Ww, K, ks, offs, qd, wd, sel), pool, st,
                                args.steps, args.warmup)
    incr = None
    if not args.no_incremental and world == 1:
        incr = measure_incremental(lsa, path, wl, offs, pool, st)
    steps = None
    if not args.no_decode_steps and world == 1:
        steps = measure_decode_steps(lsa, path, wl, offs, qd, wd, st)
    gold = None
    if not args.no_golden and world == 1:
        gold = measure_golden(lsa, device)
    trn = None
    if not args.no_train and world == 1:
        trn = measure_train(lsa, device)
    rates = None
    if not args.no_fetch_rates and world == 1:
        del path
        torch.cuda.empty_cache()
        rates = measure_fetch_rates(lsa, device, skip=(wl.name,))
        rates[wl.name] = head_rates

    result = None
    if rank == 0:
        peaks = load_peaks()
        alg = algorithmic(wl, fetched)
        ms = elapsed_ms / args.steps
        value = job_throughput(world, wl.L * T, args.steps, elapsed_ms)
        sel_ms = stage_ms[1]
        score_gbs = alg["score_bytes"] / (sel_ms * 1e-3) / 1e9
        traffic, traffic_src = score_traffic(wl)
        rooflines = {
            "project": {"bound": "hbm", "achieved": alg["proj_bytes"] / (stage_ms[0] * 1e-3) / 1e9,
                        "peak": peaks["hbm_gbs"], "unit": "GB/s", "ms": stage_ms[0]},
            "score_select": {"bound": "hbm", "achieved": score_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "ms": sel_ms},
            "fetch_rows": {"bound": "host_link", "achieved": alg["gather_host_bytes"] / (stage_ms[4] * 1e-3) / 1e9,
                           "peak": h2d, "unit": "GB/s", "ms": stage_ms[4],
                           "peak_note": "pinned host->device cudaMemcpy measured in this run",
                           "note": "second stream, overlapping the keys gather and the Top-k"},
            "fetch_keys": {"bound": "hbm", "achieved": alg["gather_key_bytes"] / (stage_ms[2] * 1e-3) / 1e9,
                           "peak": peaks["hbm_gbs"], "unit": "GB/s", "ms": stage_ms[2]},
            "lightning_topk": {"bound": "tensor", "achieved": alg["topk_flops"] / (stage_ms[3] * 1e-3) / 1e12,
                               "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s", "ms": stage_ms[3],
                               "peak_note": "sustained bf16 GEMM (timed inside the step)"},
        }
        for r in rooflines.values():
            r["frac"] = r["achieved"] / r["peak"]
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": {"fp8": "fp8_e4m3 keys / bf16 queries", "bf16": "bf16", "f32": "f32"}[wl.kdtype],
            "dtype_detail": f"keys {wl.kdtype}, queries/weights {wl.dtype}, fp32 accumulation",
            "data": "synthetic (seeded; shapes of a 1M-token context, 4:1 compression)",
            "config": workload_config(wl, args.threshold, world),
            "fetch_rate": fetched / T,
            "fetch_rates": rates if rates is not None else {wl.name: head_rates},
            "tau_window_ms": ms,
            "stages_ms": {"project": stage_ms[0], "score_select": stage_ms[1], "fetch_keys": stage_ms[2],
                          "lightning_topk": stage_ms[3], "fetch_rows (overlapped)": stage_ms[4],
                          "window": stage_ms[5]},
            "score_select_entries_per_s": world * wl.L * T / (sel_ms * 1e-3),
            "roofline": dict(kernel="score_select (index score + threshold + OR + compaction, one stream)",
                             bound="hbm", achieved=score_gbs, peak=peaks["hbm_gbs"], unit="GB/s",
                             frac=score_gbs / peaks["hbm_gbs"], frac_of_nominal_8tbs=score_gbs / 8000.0,
                             traffic=traffic,
                             traffic_note=None if traffic is None else
                             "ncu DRAM bytes of %s, scaled by entries" % traffic_src,
                             bytes_per_launch=alg["score_bytes"], peak_source=peaks["source"]),
            "rooflines": rooflines,
            "gpu_launches": launches,
            "clocks": clk,
            "e2e": e2e,
            "steady_window": steady,
            "incremental_fetch": None if incr is None else dict(incr, full_fetch_ms=stage_ms[4]),
            "decode_steps": steps,
            "golden_labels": gold,
            "train_step": trn,
        }
    pool.free()
    return result


def main():
    args = parse_args()
    rank, world, local = dist_env()

    if args.impl == "reference":
        if rank != 0:
            return 0
        import oracle
        wl = rank_workload(args.workload, 0, args.batch)
        # about two minutes of oracle work in total (~130 us per entry on 8 cores, whole path)
        n = args.cpu_sample or int(min(65536, max(2048, 120.0 / (args.steps + args.warmup) / 130e-6)))
        sw = oracle_sample_workload(wl, n)
        inp = synth.make_inputs(sw)
        for _ in range(args.warmup):
            oracle_step(oracle, sw, inp)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle_step(oracle, sw, inp)
        el = time.perf_counter() - t0
        value = sw.L * sw.total_S * args.steps / el
        cb = {"value": value, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
              "sample": f"one sequence of {sw.total_S} entries x {sw.L} layers of {wl.name} per step, whole path"}
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic", "config": workload_config(wl, args.threshold, world),
                          "cpu_baseline": cb,
                          "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return 0

    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    device = torch.device("cuda", local)
    if args.only:
        import sparse_kv_cache_memoryindexer_b200 as lsa
        torch.cuda.set_device(device)
        if args.only == "golden":
            res = measure_golden(lsa, device)
        elif args.only == "train":
            res = measure_train(lsa, device)
        else:
            res = measure_decode_only(lsa, device, args)
        print(json.dumps(dict(res, only=args.only)), flush=True)
        return 0
    if world > 1:
        torch.cuda.set_device(device)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    try:
        res = run_lsa(args, rank, world, device)
        if rank == 0:
            if not args.no_cpu_baseline and world == 1:
                res["cpu_baseline"] = cpu_baseline(synth.workload(args.workload), args.cpu_sample or 65536)
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

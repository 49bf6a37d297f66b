"""Numpy models of the two Top-k selects' steps against a plain sort (key descending, ties to the
smaller slot), on the CPU.

Decode-step select (csrc/step_select.cuh): over chunks of 2,048 candidates, four radix passes of 8
bits pick the k-th key K (per-chunk histograms added into the query's, the digit chosen by an
exclusive scan from the top), then every chunk writes its candidates above K in slot order and the
first want_eq candidates equal to K after them, and a final sort orders the k survivors.  With at
most k candidates the select takes every candidate whatever its key, including a key that orders
as 0.

Batched select (csrc/topk.cuh, k_topk_select): a 12-bit histogram of all keys gives the bucket of
the k-th key; keys of higher buckets are selected in slot order and the bucket's keys are staged
(at most SEL_CAP of them) for two 10-bit passes; a crowded bucket takes three 8/8/4-bit passes over
all keys instead.

The cases cover heavy ties in every digit, all-equal keys, keys of 0, k at and above the candidate
count, and empty queries.
"""
import zlib

import numpy as np
import pytest

CH = 2048


def select_model(u, k):
    """u: uint32 order-preserving keys of one query's candidates (slot order); returns the selected
    slots in output order."""
    nc = u.size
    remaining = k if nc > k else 0
    n_gt = 0 if nc > k else nc
    prefix = 0
    chunks = [(j0, min(nc, j0 + CH)) for j0 in range(0, nc, CH)]
    for ps in range(4):
        if remaining == 0:
            break
        shift = 24 - 8 * ps
        pmask = 0 if ps == 0 else (~((1 << (32 - 8 * ps)) - 1)) & 0xFFFFFFFF
        g = np.zeros(256, dtype=np.int64)
        for j0, j1 in chunks:
            uu = u[j0:j1]
            m = (uu & pmask) == prefix
            g += np.bincount((uu[m] >> shift) & 255, minlength=256)
        h = g[::-1]                       # thread t holds bin 255 - t
        incl = np.cumsum(h)
        above = incl - h
        chosen = np.nonzero((h > 0) & (above < remaining) & (incl >= remaining))[0]
        assert chosen.size == 1
        t = int(chosen[0])
        prefix |= (255 - t) << shift
        remaining -= int(above[t])
        n_gt += int(above[t])
    K, want_eq = prefix, remaining
    take_all = want_eq == 0               # nc <= k: every candidate, whatever its key
    out = {}
    cg = ce = 0
    for j0, j1 in chunks:
        for j in range(j0, j1):
            if take_all or u[j] > K:
                out[cg] = j
                cg += 1
            elif u[j] == K:
                if ce < want_eq:
                    out[n_gt + ce] = j
                ce += 1
    nsel = min(nc, k)
    assert cg == n_gt and len(out) == nsel
    slots = np.array([out[i] for i in range(nsel)], dtype=np.int64)
    order = np.lexsort((slots, -u[slots].astype(np.int64)))
    return slots[order]


def plain_sort(u, k):
    order = np.lexsort((np.arange(u.size), -u.astype(np.int64)))
    return order[:min(k, u.size)]


def keys(rng, kind, nc):
    if kind == "random":
        return rng.integers(0, 2 ** 32, nc, dtype=np.uint64).astype(np.uint32)
    if kind == "ties_every_digit":
        return rng.integers(0, 4, nc).astype(np.uint32) * np.uint32(0x01010101)
    if kind == "ties_low_digits":
        return (0x80000000 + rng.integers(0, 16, nc)).astype(np.uint32)
    if kind == "all_equal":
        return np.full(nc, 0x3F800000, dtype=np.uint32)
    if kind == "zeros_and_ones":
        return rng.integers(0, 2, nc).astype(np.uint32)
    return rng.standard_normal(nc).astype(np.float32).view(np.uint32) ^ np.uint32(0x80000000)


@pytest.mark.parametrize("kind", ["random", "ties_every_digit", "ties_low_digits", "all_equal", "zeros_and_ones",
                                  "float"])
def test_select_model_equals_plain_sort(kind):
    rng = np.random.default_rng(zlib.crc32(kind.encode()))
    for nc in (0, 1, 5, 100, 2047, 2048, 2049, 5000, 9000):
        for k in (1, 7, 64, 2048, 4096):
            u = keys(rng, kind, nc)
            assert np.array_equal(select_model(u, k), plain_sort(u, k)), (kind, nc, k)


def test_few_candidates_keep_a_zero_key():
    # with at most k candidates, a candidate whose key orders as 0 is still selected
    u = np.array([5, 0, 9, 0], dtype=np.uint32)
    assert select_model(u, 8).tolist() == [2, 0, 1, 3]
    assert select_model(u, 4).tolist() == [2, 0, 1, 3]
    assert select_model(np.zeros(0, dtype=np.uint32), 4).size == 0


# ------------------------------------------------------------------ batched select (csrc/topk.cuh)

def _find_bin(hist, want):
    """Bin holding the want-th largest key (bins scanned from the top) and the keys above it."""
    above = 0
    for b in range(hist.size - 1, -1, -1):
        if above + hist[b] >= want:
            return b, above
        above += int(hist[b])
    raise AssertionError("want exceeds the histogram's total")


def batched_select_model(u, k, cap=4096):
    """The batched call's select (k_topk_select): a 12-bit histogram, the k-th key's bucket staged
    (at most `cap` keys) for two 10-bit passes, or three 8/8/4-bit passes over all keys when the
    bucket is crowded; returns the selected slots in output order."""
    F = u.size
    if F <= k:
        slots = np.arange(F)
    else:
        hist = np.bincount(u >> 20, minlength=4096)
        beta, above = _find_bin(hist, k)
        sel = list(np.nonzero((u >> 20) > beta)[0])               # slot order
        assert len(sel) == above
        want = k - above
        if hist[beta] <= cap:
            staged = np.nonzero((u >> 20) == beta)[0]             # slot order
            passes = [(10, 1023), (0, 1023)]
            pool = staged
        else:
            passes = [(12, 255), (4, 255), (0, 15)]
            pool = np.arange(F)
        prefix, pmask, remaining = beta << 20, 0xFFF00000, want
        for shift, bins in passes:
            m = (u[pool] & pmask) == prefix
            h = np.bincount((u[pool][m] >> shift) & bins, minlength=1024)
            d, ab = _find_bin(h, remaining)
            prefix |= d << shift
            remaining -= ab
            pmask |= bins << shift
        inb = pool[(u[pool] >> 20) == beta]
        gt = [j for j in inb if u[j] > prefix]
        eq = [j for j in inb if u[j] == prefix][:remaining]
        assert len(gt) == want - remaining
        slots = np.array(sel + gt + eq, dtype=np.int64)
    order = np.lexsort((slots, -u[slots].astype(np.int64)))
    return slots[order]


@pytest.mark.parametrize("kind", ["random", "ties_every_digit", "ties_low_digits", "all_equal", "zeros_and_ones",
                                  "float"])
@pytest.mark.parametrize("cap", [4096, 16])
def test_batched_select_model_equals_plain_sort(kind, cap):
    rng = np.random.default_rng(zlib.crc32((kind + "batched").encode()))
    for nc in (0, 1, 100, 2047, 2049, 5000, 20000):
        for k in (1, 7, 512, 2048, 4096):
            u = keys(rng, kind, nc)
            assert np.array_equal(batched_select_model(u, k, cap), plain_sort(u, k)), (kind, nc, k, cap)

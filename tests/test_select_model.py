"""Numpy models of the two Top-k selects' steps against a plain sort (key descending, ties to the
smaller slot), on the CPU.

Both selects bucket a query's order-preserving score keys u over the query's own key range:
bucket(u) = (u - umin) >> shift, with the smallest shift that leaves at most 4,096 buckets.

Decode-step select (csrc/step_select.cuh): over chunks of 2,048 candidates, a histogram of the
buckets gives the bucket of the k-th largest key; keys of higher buckets go to the selection and the
bucket's keys to a stage, both in an arbitrary order (the model shuffles them), because every key
carries its slot: key64 = (score key << 32) | ~slot orders by score, then smaller slot, and no two
keys are equal.  The bucket's largest keys come from a sort (at most SCAP staged keys) or, for a
crowded bucket, a radix select over the stage on key64 - (umin << 32), 8 bits at a time below the
bucket's bits, stopping once a digit holds exactly the keys still wanted; one sort orders the k
keys.  With at most k candidates the select takes every candidate whatever its key, including a key
that orders as 0.

Batched select (csrc/topk.cuh, k_topk_select): the same histogram over all keys gives the bucket of
the k-th key; keys of higher buckets and the bucket's keys (at most SEL_CAP of them) are appended in
any order, and the stage sorted by 64-bit key gives the bucket's largest keys; a crowded bucket
takes radix passes of up to 8 bits over u - umin below the bucket's bits and an ordered pass
instead.

The cases cover heavy ties in every digit, all-equal keys, keys of 0, a narrow and a wide key range
(one outlier far above the rest), k at and above the candidate count, and empty queries.
"""
import zlib

import numpy as np
import pytest

CH = 2048


def _find_bin(hist, want):
    """Bin holding the want-th largest key (bins scanned from the top) and the keys above it."""
    above = 0
    for b in range(hist.size - 1, -1, -1):
        if above + hist[b] >= want:
            return b, above
        above += int(hist[b])
    raise AssertionError("want exceeds the histogram's total")


def key64(u):
    """(score key << 32) | ~slot: larger score first, then smaller slot; no two keys equal."""
    slots = np.arange(u.size, dtype=np.uint64)
    return (u.astype(np.uint64) << np.uint64(32)) | (~slots & np.uint64(0xFFFFFFFF))


def sel_range(u):
    """(umin, shift) of a query's keys: the smallest shift leaving at most 4,096 buckets."""
    umin, umax = int(u.min()), int(u.max())
    return umin, max(0, (umax - umin).bit_length() - 12)


def sel_bucket(u, umin, shift):
    return np.minimum((u.astype(np.int64) - umin) >> shift, 4095)


def select_model(u, k, scap=8192, seed=0):
    """The decode-step select (k_ss_hist12, k_ss_write and its final step): bucket histogram over the
    query's key range, keys of higher buckets and of the k-th key's bucket appended in an arbitrary
    order (shuffled here), the bucket's want largest keys by a sort (at most scap keys) or a radix
    select over the stage, then one sort of the k keys; returns the selected slots in output order."""
    rng = np.random.default_rng(seed)
    nc = u.size
    kk = key64(u)
    if nc <= k:
        slots = rng.permutation(nc)
    else:
        umin, shift = sel_range(u)
        bk = sel_bucket(u, umin, shift)
        hist = np.bincount(bk, minlength=4096)
        beta, above = _find_bin(hist, k)
        gt = rng.permutation(np.nonzero(bk > beta)[0])
        staged = rng.permutation(np.nonzero(bk == beta)[0])
        assert gt.size == above
        want = k - above
        if staged.size <= scap:
            top = staged[np.lexsort((staged, -u[staged].astype(np.int64)))][:want]
        else:
            v = kk[staged] - (np.uint64(umin) << np.uint64(32))
            prefix = np.uint64(beta << shift) << np.uint64(32)
            pmask = np.uint64((0xFFFFFFFFFFFFFFFF << (32 + shift)) & 0xFFFFFFFFFFFFFFFF)
            rem, pos = want, 32 + shift
            while pos > 0:
                wb = min(8, pos)
                sh = pos - wb
                dm = np.uint64((1 << wb) - 1)
                m = (v & pmask) == prefix
                h = np.bincount(((v[m] >> np.uint64(sh)) & dm).astype(np.int64), minlength=256)
                d, ab = _find_bin(h, rem)
                prefix |= np.uint64(d) << np.uint64(sh)
                pmask |= dm << np.uint64(sh)
                rem -= ab
                pos = sh
                if h[d] == rem:
                    break
            top = staged[v >= prefix]
            assert top.size == want
        slots = np.concatenate([gt, top]).astype(np.int64)
    order = np.argsort(kk[slots])[::-1]          # key descending: score descending, slot ascending
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
    if kind == "narrow_with_outlier":  # scores of one binade and one entry far above them
        v = (100.0 + rng.standard_normal(nc)).astype(np.float32)
        if nc:
            v[rng.integers(0, nc)] = 1e6
        return v.view(np.uint32) ^ np.uint32(0x80000000)
    return rng.standard_normal(nc).astype(np.float32).view(np.uint32) ^ np.uint32(0x80000000)


@pytest.mark.parametrize("kind", ["random", "ties_every_digit", "ties_low_digits", "all_equal", "zeros_and_ones",
                                  "narrow_with_outlier", "float"])
@pytest.mark.parametrize("scap", [8192, 16])
def test_select_model_equals_plain_sort(kind, scap):
    rng = np.random.default_rng(zlib.crc32(kind.encode()))
    for nc in (0, 1, 5, 100, 2047, 2048, 2049, 5000, 9000):
        for k in (1, 7, 64, 2048, 4096):
            u = keys(rng, kind, nc)
            assert np.array_equal(select_model(u, k, scap, seed=nc + k), plain_sort(u, k)), (kind, nc, k, scap)


def test_few_candidates_keep_a_zero_key():
    # with at most k candidates, a candidate whose key orders as 0 is still selected
    u = np.array([5, 0, 9, 0], dtype=np.uint32)
    assert select_model(u, 8).tolist() == [2, 0, 1, 3]
    assert select_model(u, 4).tolist() == [2, 0, 1, 3]
    assert select_model(np.zeros(0, dtype=np.uint32), 4).size == 0


# ------------------------------------------------------------------ batched select (csrc/topk.cuh)

def batched_select_model(u, k, cap=4096, seed=0):
    """The batched call's select (k_topk_select): a histogram over the query's key range gives the
    bucket beta of the k-th key; keys of higher buckets and (at most `cap`) keys of bucket beta are
    appended in any order (shuffled here), the stage sorted by 64-bit key gives the bucket's largest
    keys; a crowded bucket takes radix passes over u - umin below the bucket's bits and an ordered
    pass; returns the selected slots in output order."""
    rng = np.random.default_rng(seed)
    F = u.size
    kk = key64(u)
    if F <= k:
        slots = rng.permutation(F)
    else:
        umin, shift = sel_range(u)
        bk = sel_bucket(u, umin, shift)
        hist = np.bincount(bk, minlength=4096)
        beta, above = _find_bin(hist, k)
        sel = rng.permutation(np.nonzero(bk > beta)[0])
        assert sel.size == above
        want = k - above
        if hist[beta] <= cap:
            staged = rng.permutation(np.nonzero(bk == beta)[0])
            top = staged[np.argsort(kk[staged])[::-1]][:want]
        else:
            d_all = u.astype(np.int64) - umin
            dprefix, dmask, remaining, pos = beta << shift, (0xFFFFFFFF << shift) & 0xFFFFFFFF, want, shift
            while pos > 0:
                wb = min(8, pos)
                sh = pos - wb
                bins = (1 << wb) - 1
                m = (d_all & dmask) == dprefix
                h = np.bincount((d_all[m] >> sh) & bins, minlength=1024)
                d, ab = _find_bin(h, remaining)
                dprefix |= d << sh
                remaining -= ab
                dmask |= bins << sh
                pos = sh
            prefix = umin + dprefix
            inb = np.arange(F)[bk == beta]
            gt = [j for j in inb if u[j] > prefix]
            eq = [j for j in inb if u[j] == prefix][:remaining]
            assert len(gt) == want - remaining
            top = np.array(gt + eq, dtype=np.int64)
        slots = np.concatenate([sel, top]).astype(np.int64)
    order = np.argsort(kk[slots])[::-1]
    return slots[order]


@pytest.mark.parametrize("kind", ["random", "ties_every_digit", "ties_low_digits", "all_equal", "zeros_and_ones",
                                  "narrow_with_outlier", "float"])
@pytest.mark.parametrize("cap", [4096, 16])
def test_batched_select_model_equals_plain_sort(kind, cap):
    rng = np.random.default_rng(zlib.crc32((kind + "batched").encode()))
    for nc in (0, 1, 100, 2047, 2049, 5000, 20000):
        for k in (1, 7, 512, 2048, 4096):
            u = keys(rng, kind, nc)
            assert np.array_equal(batched_select_model(u, k, cap, seed=nc + k), plain_sort(u, k)), (kind, nc, k, cap)


# ------------------------------------------------------------------ block sort (csrc/common.cuh)

def block_sort_desc_model(v, nw=32):
    """block_sort_desc_u64: bitonic sort, strides >= 64 through shared memory, strides below 64 in
    each warp's 64 keys (two per lane, partners by shuffle); v: uint64 array, len a power of two
    >= 64.  Returns the sorted copy."""
    v = v.copy()
    n = v.size
    size = 2
    while size <= n:
        stride = size >> 1
        while stride >= 64:
            t = np.arange(n // 2)
            lo = 2 * t - (t & (stride - 1))
            hi = lo + stride
            desc = (lo & size) == 0
            a, c = v[lo].copy(), v[hi].copy()
            swap = (a < c) == desc
            v[lo] = np.where(swap, c, a)
            v[hi] = np.where(swap, a, c)
            stride >>= 1
        for blk in range(n // 64):
            lane = np.arange(32)
            e0 = blk * 64 + 2 * lane
            a, b = v[e0].copy(), v[e0 + 1].copy()
            desc = (e0 & size) == 0
            st = min(size >> 1, 32)
            while st >= 2:
                m = st >> 1
                low = (e0 & st) == 0
                pa, pb = a[lane ^ m], b[lane ^ m]
                keep_max = low == desc
                a = np.where(keep_max, np.maximum(a, pa), np.minimum(a, pa))
                b = np.where(keep_max, np.maximum(b, pb), np.minimum(b, pb))
                st >>= 1
            swap = (a < b) == desc
            a, b = np.where(swap, b, a), np.where(swap, a, b)
            v[e0], v[e0 + 1] = a, b
        size <<= 1
    return v


@pytest.mark.parametrize("n", [64, 128, 256, 2048, 8192])
def test_block_sort_model_sorts(n):
    rng = np.random.default_rng(n)
    for kind in ("random", "ties", "zeros"):
        if kind == "random":
            v = rng.integers(0, 2 ** 63, n, dtype=np.uint64)
        elif kind == "ties":
            v = rng.integers(0, 5, n).astype(np.uint64) << np.uint64(40)
        else:
            v = np.zeros(n, dtype=np.uint64)
            v[: n // 3] = rng.integers(1, 2 ** 40, n // 3, dtype=np.uint64)
        assert np.array_equal(block_sort_desc_model(v), np.sort(v)[::-1]), (n, kind)

"""Numpy models of the two Top-k selects' steps against a plain sort (key descending, ties to the
smaller slot), on the CPU.

Both selects bucket a query's scores linearly over the query's own score range:
bucket = floor((y - ymin) * 4096 / (ymax - ymin)) in fp32, clamped to [0, 4096), NaN to the end its
key sorts to; the bucket never decreases along the key order.

Decode-step select (csrc/step_select.cuh): over chunks of 2,048 candidates, a histogram of the
buckets gives the bucket of the k-th largest key; keys of higher buckets go to the selection and the
bucket's keys to a stage, both in an arbitrary order (the model shuffles them), because every key
carries its slot: key64 = (score key << 32) | ~slot orders by score, then smaller slot, and no two
keys are equal.  The bucket's largest keys come from a sort (at most SCAP staged keys) or, for a
crowded bucket, a radix select over the stage's 64-bit keys, 8 bits at a time from the top, stopping
once a digit holds exactly the keys still wanted; one sort orders the k
keys.  With at most k candidates the select takes every candidate whatever its key, including a key
that orders as 0.

Batched select (csrc/topk.cuh, k_topk_select): the range is that of the scores that are not NaN;
the same histogram over all keys gives the bucket of the k-th key; keys of higher buckets and the bucket's keys (at most SEL_CAP of them) are appended in
any order, and the stage sorted by 64-bit key gives the bucket's largest keys; a crowded bucket
takes four radix passes of 8 bits over the bucket's keys and an ordered pass instead.

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


def _ordered_to_float(u):
    u = np.asarray(u, dtype=np.uint32)
    b = np.where(u & np.uint32(0x80000000), u & np.uint32(0x7FFFFFFF), ~u).astype(np.uint32)
    return b.view(np.float32)


def sel_range(u):
    """(ymin, scale) of a query's keys: 4,096 buckets linear in the score over [ymin, ymax]."""
    ymin = _ordered_to_float(np.array([u.min()]))[0]
    with np.errstate(invalid="ignore", over="ignore"):  # NaN / infinite ends, spans below 2^-114
        span = np.float32(_ordered_to_float(np.array([u.max()]))[0] - ymin)
        scale = np.float32(np.float32(4096.0) / span) if span > 0 else np.float32(0.0)
    return ymin, scale


def sel_range_f(u):
    """The batched select's (ymin, scale): the smallest and largest scores that are not NaN (fminf /
    fmaxf over the scores; none: +inf and -inf, so every score falls into bucket 0 or its NaN end)."""
    y = _ordered_to_float(u)
    y = y[~np.isnan(y)]
    ymin = np.float32(y.min()) if y.size else np.float32(np.inf)
    ymax = np.float32(y.max()) if y.size else np.float32(-np.inf)
    with np.errstate(invalid="ignore", over="ignore"):
        span = np.float32(ymax - ymin)
        scale = np.float32(np.float32(4096.0) / span) if span > 0 else np.float32(0.0)
    return ymin, scale


def sel_bucket(u, ymin, scale):
    y = _ordered_to_float(u)
    with np.errstate(invalid="ignore", over="ignore"):
        t = (y - ymin).astype(np.float32) * scale
        bk = np.where(t >= np.float32(4095), 4095, np.where(t > 0, t, 0).astype(np.int64))
    nan = np.isnan(y)
    return np.where(nan, np.where(np.asarray(u) & np.uint32(0x80000000), 4095, 0), bk).astype(np.int64)


def order_desc_model(v, max_seg=32, seed=0):
    """order_desc: distinct 64-bit keys put in descending order by 4,096 buckets linear in the score
    over the keys' own range, scattered into their buckets' segments in any order (shuffled here),
    a key's position = its segment's start + the keys of its segment above it; a sort when a bucket
    holds more than max_seg keys.  Returns the ordered keys."""
    rng = np.random.default_rng(seed)
    if v.size == 0:
        return v
    u = (v >> np.uint64(32)).astype(np.uint32)
    ymin, scale = sel_range(u)
    bk = sel_bucket(u, ymin, scale)
    cnt = np.bincount(bk, minlength=4096)
    if cnt.max() > max_seg:
        return np.sort(v)[::-1]
    start = np.cumsum(cnt[::-1])[::-1] - cnt
    fill = start.copy()
    tmp = np.zeros(v.size, dtype=np.uint64)
    for t in rng.permutation(v.size):
        tmp[fill[bk[t]]] = v[t]
        fill[bk[t]] += 1
    out = np.zeros(v.size, dtype=np.uint64)
    tb = sel_bucket((tmp >> np.uint64(32)).astype(np.uint32), ymin, scale)
    for t in range(v.size):
        b = tb[t]
        lo = fill[b + 1] if b + 1 < 4096 else 0  # the end of the next bucket up is this one's start
        out[lo + int((tmp[lo:fill[b]] > tmp[t]).sum())] = tmp[t]
    return out


def select_model(u, k, scap=4096, seed=0):
    """The decode-step select (k_ss_write): the scorer's histogram of the top 14 bits of the score
    keys gives the bin beta of the k-th largest key; keys of higher bins and of bin beta are
    appended in an arbitrary order (shuffled here); with at most scap staged keys the selection and
    the stage are ordered together by order_desc and the first k kept, otherwise a 64-bit radix
    select picks the stage's want largest keys first; returns the selected slots in output order."""
    rng = np.random.default_rng(seed)
    nc = u.size
    kk = key64(u)
    if nc <= k:
        sel = kk[rng.permutation(nc)]
    else:
        bn = (u >> np.uint32(18)).astype(np.int64)
        hist = np.bincount(bn, minlength=1 << 14)
        beta, above = _find_bin(hist, k)
        want = k - above
        gt = kk[rng.permutation(np.nonzero(bn > beta)[0])]
        assert gt.size == above
        staged = kk[rng.permutation(np.nonzero(bn == beta)[0])]
        if staged.size <= scap:
            # the selection and the whole stage ordered together; the first k kept
            out = order_desc_model(np.concatenate([gt, staged]), seed=seed)[:k]
            return (~out & np.uint64(0xFFFFFFFF)).astype(np.int64)
        prefix, pmask = np.uint64(0), np.uint64(0)
        rem, pos = want, 64
        while pos > 0:
            wb = min(8, pos)
            sh = pos - wb
            dm = np.uint64((1 << wb) - 1)
            m = (staged & pmask) == prefix
            h = np.bincount(((staged[m] >> np.uint64(sh)) & dm).astype(np.int64), minlength=256)
            d, ab = _find_bin(h, rem)
            prefix |= np.uint64(d) << np.uint64(sh)
            pmask |= dm << np.uint64(sh)
            rem -= ab
            pos = sh
            if h[d] == rem:
                break
        top = staged[staged >= prefix]
        assert top.size == want
        sel = np.concatenate([gt, top])
    out = order_desc_model(sel, seed=seed)
    return (~out & np.uint64(0xFFFFFFFF)).astype(np.int64)


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
@pytest.mark.parametrize("scap", [4096, 16])
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
    keys; a crowded bucket takes four radix passes over the bucket's keys and an ordered pass;
    returns the selected slots in output order."""
    rng = np.random.default_rng(seed)
    F = u.size
    kk = key64(u)
    if F <= k:
        slots = rng.permutation(F)
    else:
        ymin, scale = sel_range_f(u)
        bk = sel_bucket(u, ymin, scale)
        hist = np.bincount(bk, minlength=4096)
        beta, above = _find_bin(hist, k)
        sel = rng.permutation(np.nonzero(bk > beta)[0])
        assert sel.size == above
        want = k - above
        if hist[beta] <= cap:
            staged = rng.permutation(np.nonzero(bk == beta)[0])
            top = staged[np.argsort(kk[staged])[::-1]][:want]
        else:
            prefix, pmask, remaining = 0, 0, want
            inb_mask = bk == beta
            for sh in (24, 16, 8, 0):
                m = inb_mask & ((u & np.uint32(pmask)) == prefix)
                h = np.bincount((u[m] >> np.uint32(sh)) & np.uint32(255), minlength=1024)
                d, ab = _find_bin(h, remaining)
                prefix |= d << sh
                remaining -= ab
                pmask |= 255 << sh
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


# ------------------------------------------------------------------ block sort (csrc/select_common.cuh)

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


# ------------------------------------------------------------------ selection order without a sort

def ranked_order_model(u, k, seed=0, rangef=None):
    """Both selects' ordering of the selection when no bucket above beta is large: every bucket
    above beta gets a segment of the selection (higher buckets first, each segment's start the keys
    of the buckets above it), its keys are scattered into it in any order (shuffled here), and a
    key's output position is its segment's start plus the keys of its segment above it; the k-th
    key's bucket's largest keys follow in key order.  Returns (slots in output order, largest
    segment)."""
    rng = np.random.default_rng(seed)
    kk = key64(u)
    ymin, scale = (rangef or sel_range)(u)
    bk = sel_bucket(u, ymin, scale)
    hist = np.bincount(bk, minlength=4096)
    beta, above = _find_bin(hist, k)
    start = np.zeros(4097, dtype=np.int64)       # start[b] = keys in buckets above b (b > beta)
    start[:4096] = np.cumsum(hist[::-1])[::-1] - hist
    sel = np.zeros(above, dtype=np.uint64)
    fill = start.copy()
    for j in rng.permutation(np.nonzero(bk > beta)[0]):
        sel[fill[bk[j]]] = kk[j]
        fill[bk[j]] += 1
    out = np.zeros(k, dtype=np.uint64)
    for t in range(above):
        v = sel[t]
        b = sel_bucket(np.array([v >> np.uint64(32)], dtype=np.uint32), ymin, scale)[0]
        lo = fill[b + 1] if b + 1 < 4096 else 0  # the end of the next bucket up is this one's start
        hi = fill[b]
        out[lo + int((sel[lo:hi] > v).sum())] = v
    staged = np.nonzero(bk == beta)[0]
    out[above:] = np.sort(kk[staged])[::-1][:k - above]
    slots = (~out & np.uint64(0xFFFFFFFF)).astype(np.int64)
    return slots, int(hist[beta + 1:].max()) if beta + 1 < 4096 else 0


@pytest.mark.parametrize("rangef", ["keys", "scores"])
@pytest.mark.parametrize("kind", ["random", "ties_every_digit", "ties_low_digits", "narrow_with_outlier", "float"])
def test_ranked_order_equals_plain_sort(kind, rangef):
    """rangef: the range of the keys (the decode step's order) or of the non-NaN scores (the
    batched select)."""
    rng = np.random.default_rng(zlib.crc32((kind + "ranked").encode()))
    for nc in (2049, 5000, 31000):
        for k in (1, 7, 512, 2048):
            u = keys(rng, kind, nc)
            slots, _ = ranked_order_model(u, k, seed=nc + k, rangef=sel_range if rangef == "keys" else sel_range_f)
            assert np.array_equal(slots, plain_sort(u, k)), (kind, nc, k)

"""Numpy model of the golden-label vote's bit-sliced counting (csrc/golden.cuh, k_golden_vote)
against a plain per-entry count, on the CPU.

The kernel holds, for one 32-entry word and one token, the vote count of each of the 32 entries in
bit slices: slice k is a 32-bit word whose bit e is bit k of entry e's count.  Adding a layer's
kept-bits word x is a ripple-carry add of x into the slices (t = c_k & carry; c_k ^= carry;
carry = t).  "count >= theta" is then decided slice by slice from the most significant one: with
gt = entries already known above theta and eq = entries equal to theta so far, a set bit of theta
keeps eq only where the entry's bit is set, a clear bit moves eq-and-set entries to gt and keeps eq
only where the bit is clear; the result is gt | eq.  The slices needed are those of Lc (counts never
exceed Lc); theta above Lc keeps nothing.
"""
import numpy as np
import pytest

SLICES = 8
MASK = 0xFFFFFFFF


def vote_word_model(planes, theta):
    """planes: the Lc kept-bits words of one token (ints); returns the word of entries with at
    least theta votes, as the kernel computes it."""
    Lc = len(planes)
    ns = 0
    while ns < SLICES and (Lc >> ns) != 0:
        ns += 1
    if theta > Lc:
        return 0
    c = [0] * SLICES
    for x in planes:
        carry = x
        for k in range(SLICES):
            t = c[k] & carry
            c[k] ^= carry
            carry = t
    gt, eq = 0, MASK
    for k in range(SLICES - 1, -1, -1):
        if k >= ns:
            continue
        if (theta >> k) & 1:
            eq &= c[k]
        else:
            gt |= eq & c[k]
            eq &= ~c[k] & MASK
    return (gt | eq) & MASK


def vote_word_plain(planes, theta):
    out = 0
    for e in range(32):
        votes = sum((x >> e) & 1 for x in planes)
        if votes >= theta:
            out |= 1 << e
    return out


@pytest.mark.parametrize("Lc", [1, 2, 3, 7, 8, 21, 31, 32, 64, 255])
def test_vote_model_equals_plain_count(Lc):
    rng = np.random.default_rng(Lc)
    for density in (0.05, 0.5, 0.95):
        for _ in range(4):
            planes = [int(w) for w in (rng.random((Lc, 32)) < density).astype(np.uint64) @ (1 << np.arange(32, dtype=np.uint64))]
            for theta in sorted({1, 2, 3, Lc // 2 + 1, Lc, Lc + 1}):
                if theta < 1:
                    continue
                assert vote_word_model(planes, theta) == vote_word_plain(planes, theta), (Lc, density, theta)


def test_vote_model_edges():
    # every layer keeps every entry: all counts are Lc
    assert vote_word_model([MASK] * 21, 21) == MASK
    assert vote_word_model([MASK] * 21, 22) == 0
    # no layer keeps anything
    assert vote_word_model([0] * 21, 1) == 0
    # entry 0 kept by five layers, entry 1 by three
    planes = [0b01] * 2 + [0b11] * 3
    assert vote_word_model(planes, 3) == 0b11 and vote_word_model(planes, 4) == 0b01
    # counts that fill every slice (Lc = 255)
    assert vote_word_model([1] * 255, 255) == 1

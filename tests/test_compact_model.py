"""Model of the compaction's writes (csrc/score_select.cuh, k_compact) on the CPU: from the fetch
words of a sequence's tiles (4 x 32 bits per 128-entry tile), the list positions (tile start from
the prefix of the popcounts, then p + popc(word & lanes below) for each set bit, word by word) and
the byte mask (4 bytes per lane packed from a nibble of its word) equal the plain ascending list of
set entries and the plain 0/1 mask, for ragged sequence lengths.
"""
import numpy as np
import pytest

TILE = 128


def compact_model(words, S):
    """words: [tiles][4] uint32 fetch words of one sequence; returns (list, mask)."""
    ntiles = words.shape[0]
    counts = [sum(bin(int(w)).count("1") for w in words[t]) for t in range(ntiles)]
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]]).astype(int) if ntiles else np.zeros(0, int)
    out = np.full(int(sum(counts)), -1, dtype=np.int64)
    mask = np.full(S, 255, dtype=np.uint8)
    for t in range(ntiles):
        p = int(starts[t])
        s0 = t * TILE
        for k in range(4):
            wk = int(words[t, k])
            for lane in range(32):
                if (wk >> lane) & 1:
                    out[p + bin(wk & ((1 << lane) - 1)).count("1")] = s0 + 32 * k + lane
            p += bin(wk).count("1")
        for lane in range(32):  # the packed mask bytes
            wl = int(words[t, lane // 8])
            nib = (wl >> (4 * (lane & 7))) & 0xF
            packed = (nib & 1) | ((nib & 2) << 7) | ((nib & 4) << 14) | ((nib & 8) << 21)
            for q in range(4):
                e = s0 + 4 * lane + q
                if e < S:
                    mask[e] = (packed >> (8 * q)) & 1
    return out, mask


@pytest.mark.parametrize("S", [1, 127, 128, 129, 1000, 4096])
def test_compaction_model_equals_plain(S):
    rng = np.random.default_rng(S)
    ntiles = (S + TILE - 1) // TILE
    bits = rng.random(ntiles * TILE) < 0.135
    bits[S:] = False  # entries past the sequence's end are never fetched
    words = np.zeros((ntiles, 4), dtype=np.uint64)
    for i in np.nonzero(bits)[0]:
        words[i // TILE, (i % TILE) // 32] |= np.uint64(1) << np.uint64(i % 32)
    lst, mask = compact_model(words, S)
    assert np.array_equal(lst, np.nonzero(bits[:S])[0])
    assert np.array_equal(mask, bits[:S].astype(np.uint8))

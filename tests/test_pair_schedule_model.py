"""Model of the CTA-pair score kernel's work split (csrc/score_pair.cuh, k_score_pair) on the CPU:
every 128-entry tile of every sequence is scored exactly once, by the CTA whose rank matches its
position in its pair job, and the key bytes the leader expects per job match the loads issued.

A job is two consecutive tiles of one sequence (ceil(tiles / 2) jobs per sequence, their prefix
pstart); pair pi of npair takes jobs [pi NJ / npair, (pi + 1) NJ / npair); the rank-r CTA's tile
in job j of sequence b is 2 (j - pstart[b]) + r, loaded when it exists; the leader expects one or
two tiles' bytes; the sequence of job j is found by walking pstart forward (sequences without jobs
are skipped).
"""
import numpy as np
import pytest

TILE = 128


class Tracker:
    """The kernel's forward walk over pstart (one per role and CTA; jobs visited in order)."""

    def __init__(self, pstart):
        self.p = pstart
        self.b, self.next = 0, -1
        self.first = 0

    def of(self, j):
        if self.next < 0 or self.next <= j:
            if self.next < 0:
                self.next = self.p[1]
            while self.next <= j:
                self.b += 1
                self.next = self.p[self.b + 1]
            self.first = self.p[self.b]
        return self.b


def schedule(S, npair):
    tiles = [(s + TILE - 1) // TILE for s in S]
    pstart = [0]
    for n in tiles:
        pstart.append(pstart[-1] + (n + 1) // 2)
    NJ = pstart[-1]
    seen = {}
    for pi in range(npair):
        j0, j1 = pi * NJ // npair, (pi + 1) * NJ // npair
        for rank in (0, 1):
            tr = Tracker(pstart)
            for j in range(j0, j1):
                b = tr.of(j)
                assert pstart[b] <= j < pstart[b + 1]
                base = 2 * (j - tr.first)
                tl = base + rank
                mine = tl < tiles[b]
                both = base + 1 < tiles[b]
                loads = sum(1 for r in (0, 1) if base + r < tiles[b])
                assert loads == (2 if both else 1)          # the leader's expected bytes / 16 KB
                if mine:
                    key = (b, tl)
                    assert key not in seen, f"tile {key} scored twice"
                    seen[key] = (pi, rank)
                    rows = [tl * TILE + q for q in range(TILE)]
                    valid = [s for s in rows if s < S[b]]
                    assert len(valid) == min(TILE, S[b] - tl * TILE)
    for b, n in enumerate(tiles):
        for t in range(n):
            assert (b, t) in seen, f"tile {(b, t)} never scored"
    return seen


@pytest.mark.parametrize("seed", range(6))
def test_every_tile_scored_once(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 80))
    S = [int(x) for x in rng.choice([0, 1, 127, 128, 129, 255, 256, 1000, 33000], size=B)]
    for npair in (1, 3, 74):
        schedule(S, npair)


def test_bench_shape_and_edges():
    schedule([262144] * 32, 74)             # 1,024 jobs per sequence, 443 per pair
    schedule([0, 0, 0], 74)                 # no tiles at all
    schedule([1], 74)                       # one job whose peer tile does not exist
    schedule([0, 129, 0, 1, 0], 2)          # empty sequences between odd ones

"""Model of how the batched select (csrc/topk.cuh, ScoreRow) and the golden-label kernel
(csrc/golden.cuh) split a row of fp32 values into 16-byte vectors and lone entries, on the CPU:
every entry of the row is read exactly once, no read leaves the row, and every vector starts on a
16-byte boundary, for every alignment of the row's start and every length.

head = min((4 - (address / 4) mod 4) mod 4, F) entries before the first boundary; nvec = (F - head)
/ 4 whole vectors from there; the F - (head + 4 nvec) entries after them; thread t < head takes entry
t, thread head + i takes entry head + 4 nvec + i.
"""
import pytest

THREADS = 1024  # the select's block (the golden kernel's 256 threads take the same entries)


def split(addr_floats, F, threads=THREADS):
    head = min((4 - addr_floats % 4) % 4, F)
    nvec = (F - head) // 4
    tail0 = head + 4 * nvec
    seen = []
    for v in range(nvec):
        start = head + 4 * v
        assert (addr_floats + start) % 4 == 0  # 16-byte aligned vector
        seen.extend(range(start, start + 4))
    for t in range(threads):
        if t < head:
            seen.append(t)
        elif t < head + (F - tail0):
            seen.append(tail0 + (t - head))
    return seen


@pytest.mark.parametrize("align", [0, 1, 2, 3])
def test_every_entry_read_once(align):
    for F in list(range(0, 40)) + [1023, 1024, 1025, 4099, 31000, 32768]:
        seen = split(align, F)
        assert sorted(seen) == list(range(F)), (align, F)
        assert all(0 <= s < F for s in seen)


def test_at_most_six_lone_entries():
    for align in range(4):
        for F in range(0, 64):
            head = min((4 - align % 4) % 4, F)
            nvec = (F - head) // 4
            assert head + (F - head - 4 * nvec) <= 6

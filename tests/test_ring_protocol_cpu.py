"""The decode kernel's byte-ring protocol, restated and model-checked on the
CPU.

The producer lane places each chunk (a weight chunk or an attention tile)
right after the previous one, or at 0 when it would run past the end of the
ring, and before issuing the copy waits, oldest first, until fewer than 16
chunks are live and no live chunk overlaps the new range (the kernel's
`ring_place` and `Producer::acquire`).  The consumers walk the same chunk
sequence and recompute every offset themselves.  Random interleavings of the
two sides must never let a copy land on bytes a consumer has not released,
never reuse one of the 16 barrier pairs while its chunk is live, and always
give both sides the same offsets.  Checking only the oldest live chunk for
overlap is a plausible simplification that is wrong when both the live
region and the new chunk wrap; the model must catch it.
"""
import random

import pytest

N_BARS = 16


def place(wend: int, size: int, ring: int):
    off = wend if wend + size <= ring else 0
    return off, off + size


def producer(sizes, ring, shared, check_all=True):
    """Generator: one yield per step that may block on the consumers."""
    idx = cons = 0
    wend = 0
    live = [(0, 0)] * N_BARS
    for size in sizes:
        off, wend = place(wend, size, ring)
        while cons < idx:
            blocked = idx - cons >= N_BARS
            span = range(cons, idx) if check_all else range(cons, cons + 1)
            for j in span:
                if blocked:
                    break
                lo, hi = live[j % N_BARS]
                blocked = off < hi and lo < off + size
            if not blocked:
                break
            while shared["consumed"] <= cons:      # wait until chunk `cons` is released
                yield
            cons += 1
        # the copy is issued now: it must not touch any unreleased chunk
        for j in range(shared["consumed"], idx):
            lo, hi = shared["where"][j]
            assert not (off < hi and lo < off + size), ("overlap", idx, j)
        assert idx - shared["consumed"] < N_BARS, "barrier pair reused while live"
        shared["where"][idx] = (off, off + size)
        live[idx % N_BARS] = (off, off + size)
        idx += 1
        shared["issued"] = idx
        yield


def run(sizes, ring, seed, check_all=True):
    rnd = random.Random(seed)
    shared = {"consumed": 0, "issued": 0, "where": {}}
    prod = producer(sizes, ring, shared, check_all)
    finished = False
    cend = 0
    for _ in range(10 ** 6):
        if shared["consumed"] == len(sizes):
            return
        if not finished and rnd.random() < 0.5:
            try:
                next(prod)
            except StopIteration:
                finished = True
        elif shared["consumed"] < shared["issued"]:
            i = shared["consumed"]
            off, cend = place(cend, sizes[i], ring)
            assert (off, off + sizes[i]) == shared["where"][i], "consumer offset differs"
            shared["consumed"] += 1
    raise AssertionError("no progress")


def _case(seed):
    rnd = random.Random(seed)
    ring = rnd.choice([30720, 65536, 100352, 191488, 196608, 209920])
    mix = [4096, 8192, 20480, 24576, 32768, 40960, 65536]
    sizes = [min(ring // 2, rnd.choice(mix + [512 * rnd.randint(8, 128)])) for _ in range(300)]
    return sizes, ring


def test_ring_protocol_random_interleavings():
    for seed in range(600):
        sizes, ring = _case(seed)
        run(sizes, ring, seed)


def test_checking_only_the_oldest_chunk_is_caught():
    with pytest.raises(AssertionError) as e:
        for seed in range(600):
            sizes, ring = _case(seed)
            run(sizes, ring, seed, check_all=False)
    assert "overlap" in str(e.value), str(e.value)

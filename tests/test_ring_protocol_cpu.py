"""The decode kernel's byte-ring protocol, restated and model-checked on the
CPU.

The producer lane places each chunk (a weight chunk or an attention tile)
right after the previous one, or at 0 when it would run past the end of the
ring (the kernel's `ring_place`).  Besides the ring offset it keeps a
monotonic byte position that also counts the bytes skipped at each wrap, so
chunk i occupies the monotonic range [s_i, e_i) and its ring bytes are that
range modulo the ring size R.  The live chunks of a new chunk [s, e) lie in
[s_oldest, s); once the oldest live chunk starts at or after e - R they all
lie in [e - R, s), which together with [s, e) spans exactly R bytes, so none
of them shares a ring byte with the new chunk.  The producer counts chunks
as released oldest first: it waits for the oldest live chunk's release until
that chunk starts at or after e - R and fewer than 32 chunks are live
(`Producer::acquire`); one comparison per released chunk.  A GEMV stage's
chunks are released out of order -- each belongs to one consumer warp
(chunk u of the stage to warp u % 8), which computes its own chunks in
order -- and a warp learns a chunk's offset from the table the producer
writes (one slot per barrier pair) before it arms the chunk's barrier.
Random interleavings of the producer and eight warps must never let a copy
land on bytes a warp has not released, never reuse one of the 32 barrier
pairs while its chunk is live, and always hand a warp the offset its chunk
was copied to.  Two plausible slips must be caught: checking only the oldest
live chunk for overlap in ring offsets (wrong when both the live region and
the new chunk wrap), and comparing the oldest start against s - R instead of
e - R.
"""
import random

import pytest

N_BARS = 32
N_WARPS = 8


def place(wend: int, size: int, ring: int):
    off = wend if wend + size <= ring else 0
    return off, off + size


def producer(sizes, ring, shared, rule="monotonic"):
    """Generator: one yield per step that may block on the consumers.

    rule "monotonic": the kernel's rule (see the module docstring);
    "oldest_offsets": overlap of the new range with the oldest live chunk's
    ring offsets only; "start_minus_ring": the monotonic rule with s - R in
    place of e - R."""
    idx = cons = 0
    wend = 0
    head = 0                          # monotonic write position
    live = [(0, 0)] * N_BARS
    starts = [0] * N_BARS
    for size in sizes:
        prev = wend
        off, wend = place(wend, size, ring)
        if off == 0 and prev != 0:
            head += ring - prev       # bytes skipped at the wrap
        s, e = head, head + size
        head = e
        while cons < idx:
            if rule == "oldest_offsets":
                lo, hi = live[cons % N_BARS]
                blocked = idx - cons >= N_BARS or (off < hi and lo < off + size)
            else:
                bound = e - ring if rule == "monotonic" else s - ring
                blocked = idx - cons >= N_BARS or starts[cons % N_BARS] < bound
            if not blocked:
                break
            while cons not in shared["released"]:   # wait until chunk `cons` is released
                yield
            cons += 1
        # the copy is issued now: it must not touch any unreleased chunk
        unreleased = [j for j in range(idx) if j not in shared["released"]]
        for j in unreleased:
            lo, hi = shared["where"][j]
            assert not (off < hi and lo < off + size), ("overlap", idx, j)
        assert not unreleased or idx - unreleased[0] < N_BARS, "barrier pair reused while live"
        shared["where"][idx] = (off, off + size)
        shared["table"][idx % N_BARS] = off      # published before the barrier is armed
        live[idx % N_BARS] = (off, off + size)
        starts[idx % N_BARS] = s
        idx += 1
        shared["issued"] = idx
        yield


def run(sizes, ring, seed, rule="monotonic"):
    rnd = random.Random(seed)
    shared = {"released": set(), "issued": 0, "where": {}, "table": [None] * N_BARS}
    prod = producer(sizes, ring, shared, rule)
    finished = False
    nxt = list(range(N_WARPS))          # next chunk of each warp: w, w + 8, ...
    for _ in range(10 ** 6):
        if len(shared["released"]) == len(sizes):
            return
        if not finished and rnd.random() < 0.5:
            try:
                next(prod)
            except StopIteration:
                finished = True
        else:
            w = rnd.randrange(N_WARPS)
            i = nxt[w]
            if i < shared["issued"]:
                off = shared["table"][i % N_BARS]
                assert (off, off + sizes[i]) == shared["where"][i], "consumer offset differs"
                shared["released"].add(i)
                nxt[w] += N_WARPS
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


@pytest.mark.parametrize("rule", ["oldest_offsets", "start_minus_ring"])
def test_plausible_wrong_rules_are_caught(rule):
    with pytest.raises(AssertionError) as e:
        for seed in range(600):
            sizes, ring = _case(seed)
            run(sizes, ring, seed, rule=rule)
    assert "overlap" in str(e.value), str(e.value)

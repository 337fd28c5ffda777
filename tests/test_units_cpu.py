"""The GEMV work units of the decode kernel, through the host-only planning
query `kie_plan_gemv_work` (the function the kernel and its weight repack
call, compiled for the host).  A CTA's rows of a stage are cut into blocks
of nr <= 4 rows and every row's 256-weight pieces into S parts; a block's
part is one bulk copy computed by one consumer warp.  Checked on the CPU:
every unit fits a chunk, split rows fit the result slots, the blocks cover
the rows, the parts cover the pieces, the shape is the cheapest under the
documented cost model, and the 2.2B model gets the shapes the kernel's
measurements were taken with."""
import itertools
import random

import pytest

import synth
from persistent_sm_decode_monokernel_b200 import _kie, build

GRID = 148
PIECE = 256


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _kie.load_library()


def _desc(shape, max_seq=2048):
    return _kie.make_desc(shape.n_layers, shape.d_model, shape.n_heads, shape.n_kv_heads,
                          shape.head_dim, shape.ffn_dim, shape.vocab, shape.rope_base,
                          shape.rms_eps, max_seq)


def _cost(rows, kp, nr, S):
    """Busiest warp's time in piece-rows: units run one after another on
    warp u % 8; a unit of r rows and n pieces costs r*n + 0.3*n + 6 (x10)."""
    nb = -(-rows // nr)
    nmax = -(-kp // S)
    return -(-(nb * S) // 8) * (10 * nr * nmax + 3 * nmax + 60)


def _check_plan(rows, kp, nr, S, nb, slots, chunk, fp8):
    pb = PIECE * (1 if fp8 else 2)
    assert 1 <= nr <= 4 and (nr == 1 or nr <= rows)
    assert 1 <= S <= kp
    nmax = -(-kp // S)
    assert nr * nmax * pb <= chunk, "a unit is larger than a chunk"
    assert S == 1 or rows * S <= slots, "split rows need more result slots"
    assert slots >= max(256, rows)
    assert nb == -(-rows // nr) and (nb - 1) * nr < rows <= nb * nr
    # parts: base + (s < rem) pieces from s*base + min(s, rem), covering 0..kp
    base, rem = kp // S, kp % S
    firsts = [s * base + min(s, rem) for s in range(S)]
    counts = [base + (1 if s < rem else 0) for s in range(S)]
    assert firsts[0] == 0 and all(firsts[s] + counts[s] == firsts[s + 1] for s in range(S - 1))
    assert firsts[-1] + counts[-1] == kp
    # the cheapest feasible shape, first in (nr, S) order among equals
    m = chunk // pb
    best = None
    for n_r in range(1, 5):
        if n_r > 1 and n_r > rows:
            break
        for s in range(1, min(kp, 16) + 1):
            if n_r * -(-kp // s) > m:
                continue
            if s > 1 and rows * s > slots:
                break
            c = _cost(rows, kp, n_r, s)
            if best is None or c < best[0]:
                best = (c, n_r, s)
    if best is not None:
        assert (nr, S) == best[1:], (rows, kp, chunk, (nr, S), best)


def test_shapes_of_the_2p2b_model(lib):
    d = _desc(synth.WORKLOADS["l28-d2560"].shape)
    got = {st: {_kie.kie_plan_gemv_work(d, GRID, st, c)[2:4] for c in range(GRID)} for st in range(5)}
    assert got[0] <= {(3, 1), (4, 1)}        # QKV: 24-26 rows of 10 pieces, one block per warp
    assert got[1] == {(3, 1)}                 # O: 17-18 rows, six blocks of 3
    assert got[2] == {(4, 1)}                 # gate/up: 92-94 rows, 20 KB units
    assert got[3] == {(3, 4)}                 # down: 27 pieces a row in 4 parts
    assert got[4] == {(4, 1)}                 # LM head: ~340 rows
    # every CTA's units fit the default 32 KB chunk and cover its rows
    for st in range(5):
        for c in range(GRID):
            rows, kp, nr, S, nb, slots = _kie.kie_plan_gemv_work(d, GRID, st, c)
            _check_plan(rows, kp, nr, S, nb, slots, 32768, 0)


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
@pytest.mark.parametrize("chunk,fp8", [(8192, 0), (12800, 0), (32768, 0), (98304, 0),
                                       (8192, 1), (32768, 1)])
def test_plan_invariants_on_every_workload(lib, name, chunk, fp8):
    d = _desc(synth.WORKLOADS[name].shape)
    grid = min(GRID, *(_kie.kie_plan_units(d, GRID, st, GRID - 1)[1] for st in range(5)))
    rnd = random.Random(hash((name, chunk, fp8)) & 0xffff)
    for st in range(5):
        for c in rnd.sample(range(grid), min(grid, 12)):
            rows, kp, nr, S, nb, slots = _kie.kie_plan_gemv_work(d, grid, st, c, chunk, fp8)
            _check_plan(rows, kp, nr, S, nb, slots, chunk, fp8)


def test_plan_invariants_on_random_shapes(lib):
    rnd = random.Random(7)
    checked = 0
    for _ in range(60):
        kv = rnd.choice([1, 2, 4, 8])
        g = rnd.choice([1, 2, 4, 5, 8])
        hd = rnd.choice([64, 128])
        shape = synth.ModelShape(rnd.randint(1, 4), 256 * rnd.randint(1, 24), kv * g, kv, hd,
                                 256 * rnd.randint(2, 60), rnd.randint(1000, 140000))
        d = _desc(shape)
        if _kie.kie_check_desc(d) != _kie.KIE_OK:
            continue
        grid = rnd.choice([1, 7, 64, 148])
        chunk = 512 * rnd.randint(16, 200)
        fp8 = rnd.randint(0, 1)
        for st, c in itertools.product(range(5), rnd.sample(range(grid), min(grid, 4))):
            rows, kp, nr, S, nb, slots = _kie.kie_plan_gemv_work(d, grid, st, c, chunk, fp8)
            if rows == 0:
                continue
            _check_plan(rows, kp, nr, S, nb, slots, chunk, fp8)
            checked += 1
    assert checked > 300


def test_plan_query_rejects_bad_arguments(lib):
    d = _desc(synth.WORKLOADS["tiny-l2-d256"].shape, 64)
    for args in [(0, 0, 0, 32768, 0), (4, 5, 0, 32768, 0), (4, 0, 4, 32768, 0),
                 (4, 0, 0, 4096, 0), (4, 0, 0, 32768 + 100, 0), (4, 0, 0, 32768, 2)]:
        with pytest.raises(RuntimeError):
            _kie.kie_plan_gemv_work(d, *args)

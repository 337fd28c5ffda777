"""Pins of the sampling oracle (no GPU).

* The Philox4x64-10 block is checked against numpy's own implementation of
  the same generator (`numpy.random.Philox`, a separate library routine),
  which advances its 256-bit counter by one before each block.
* Gumbel-max over logits / T must draw from softmax(logits / T): empirical
  frequencies over many positions against the closed-form probabilities.
* Special cases: T -> 0 gives the greedy argmax, T <= 0 is greedy, a huge T
  makes the draw independent of the logits, uniforms stay inside (0, 1).
"""
import numpy as np
import pytest

from oracle import sampling as S

MASK = (1 << 64) - 1


def _numpy_block(counter, key):
    """numpy's Philox, positioned so its next block uses `counter`."""
    c = [int(v) for v in counter]
    # numpy adds one to the counter (with carry) before each block: start
    # one below the wanted counter
    words = c[0] | (c[1] << 64) | (c[2] << 128) | (c[3] << 192)
    words = (words - 1) % (1 << 256)
    start = [(words >> (64 * i)) & MASK for i in range(4)]
    g = np.random.Philox(counter=np.array(start, dtype=np.uint64),
                         key=np.array([int(k) for k in key], dtype=np.uint64))
    return [int(x) for x in g.random_raw(4)]


@pytest.mark.parametrize("counter,key", [
    ((0, 0, 0, 0), (0, 0)),
    ((1, 0, 0, 0), (0, 0)),
    ((MASK, MASK, MASK, MASK), (MASK, MASK)),
    ((12345, 678, 0, 0), (2024, 0)),
    ((0, 1 << 40, 7, 9), (0xDEADBEEF, 0x1234)),
    ((0x243F6A8885A308D3, 0x13198A2E03707344, 0xA4093822299F31D0, 0x082EFA98EC4E6C89),
     (0x452821E638D01377, 0xBE5466CF34E90C6C)),
])
def test_philox_block_matches_numpy(counter, key):
    assert S.philox4x64_10(counter, key) == _numpy_block(counter, key)


def test_vectorised_philox_matches_numpy():
    rng = np.random.default_rng(7)
    c0 = rng.integers(0, 1 << 63, size=64, dtype=np.uint64)
    c1 = rng.integers(0, 1 << 20, size=64, dtype=np.uint64)
    got = S.philox4x64_10_many(c0, c1, 99)
    for i in range(64):
        assert [int(x) for x in got[i]] == _numpy_block((int(c0[i]), int(c1[i]), 0, 0), (99, 0))


def test_uniform_layout_and_range():
    n = 10
    u = S.uniforms(5, 33, n)
    for i in range(n):
        w = S.philox4x64_10((i // 4, 33, 0, 0), (5, 0))[i % 4]
        assert u[i] == ((w >> 11) + 0.5) * 2.0 ** -53
    big = S.uniforms(1, np.arange(200), 4096)
    assert big.min() > 0.0 and big.max() < 1.0
    assert abs(big.mean() - 0.5) < 0.01
    # different positions and seeds give different streams
    assert not np.array_equal(S.uniforms(1, 0, 64), S.uniforms(1, 1, 64))
    assert not np.array_equal(S.uniforms(1, 0, 64), S.uniforms(2, 0, 64))


def _softmax(z):
    e = np.exp(z - z.max())
    return e / e.sum()


@pytest.mark.parametrize("T", [0.7, 1.0, 2.5])
def test_gumbel_max_draws_softmax(T):
    logits = np.array([0.5, -1.0, 2.0, 0.0, 1.2, -0.3], dtype=np.float32)
    n = 40000
    u = S.uniforms(11, np.arange(n), logits.shape[0])
    draws = np.argmax(S.perturbed_scores(logits, T, 11, np.arange(n)), axis=1)
    freq = np.bincount(draws, minlength=logits.shape[0])
    p = _softmax(logits.astype(np.float64) / T)
    chi2 = float(((freq - n * p) ** 2 / (n * p)).sum())
    assert chi2 < 35.0, (chi2, freq, n * p)       # 5 dof: p < 1e-6 at 35
    # the same draws with the wrong sign of the noise, or T multiplying
    # instead of dividing, are far from the target distribution
    wrong = np.argmax(logits.astype(np.float64) / T - S.gumbel(u), axis=1)
    fw = np.bincount(wrong, minlength=logits.shape[0])
    assert float(((fw - n * p) ** 2 / (n * p)).sum()) > 100.0
    if T != 1.0:
        wt = np.argmax(logits.astype(np.float64) * T + S.gumbel(u), axis=1)
        ft = np.bincount(wt, minlength=logits.shape[0])
        assert float(((ft - n * p) ** 2 / (n * p)).sum()) > 100.0


def test_limits():
    rng = np.random.default_rng(3)
    for pos in range(20):
        lg = rng.standard_normal(1000).astype(np.float32)
        assert S.sample_id(lg, 1e-7, 4, pos) == int(np.argmax(lg))
        assert S.sample_id(lg, 0.0, 4, pos) == int(np.argmax(lg))
        # huge T: the draw is the argmax of the uniforms alone
        assert S.sample_id(lg, 1e9, 4, pos) == int(np.argmax(S.uniforms(4, pos, 1000)))


def test_score_margin():
    assert S.score_margin(np.array([1.0, 3.0, 2.5])) == pytest.approx(0.5)
    assert S.score_margin(np.array([1.0])) == float("inf")


# ---- planted mistakes: each must make one of the pins above fail

def _philox_early_key_bump(counter, key):
    c0, c1, c2, c3 = (int(v) & MASK for v in counter)
    k0, k1 = (int(v) & MASK for v in key)
    for _ in range(10):
        k0 = (k0 + S.PHILOX_W0) & MASK
        k1 = (k1 + S.PHILOX_W1) & MASK
        p0, p1 = S.PHILOX_M0 * c0, S.PHILOX_M1 * c2
        c0, c1, c2, c3 = (p1 >> 64) ^ c1 ^ k0, p1 & MASK, (p0 >> 64) ^ c3 ^ k1, p0 & MASK
    return [c0, c1, c2, c3]


def _philox_many_swapped_multipliers(c0, c1, key0):
    saved = S.PHILOX_M0, S.PHILOX_M1
    try:
        S.PHILOX_M0, S.PHILOX_M1 = saved[1], saved[0]
        return _ORIG["philox4x64_10_many"](c0, c1, key0)
    finally:
        S.PHILOX_M0, S.PHILOX_M1 = saved


def _uniforms_no_half(seed, position, n):
    return _ORIG["uniforms"](seed, position, n) - 0.5 * 2.0 ** -53


def _uniforms_swapped_counter(seed, position, n):
    nb = (n + 3) // 4
    pos = np.asarray(position, dtype=np.uint64)
    words = S.philox4x64_10_many(pos[..., None], np.arange(nb, dtype=np.uint64), seed)
    words = words.reshape(pos.shape + (4 * nb,))[..., :n]
    return ((words >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53


def _gumbel_wrong_sign(u):
    return np.log(-np.log(u))


def _scores_times_t(logits, temperature, seed, position):
    lg = np.asarray(logits, dtype=np.float64)
    return lg * float(temperature) + S.gumbel(S.uniforms(seed, position, lg.shape[0]))


def _sample_id_argmin(logits, temperature, seed, position):
    if temperature <= 0:
        return int(np.argmin(np.asarray(logits)))
    return int(np.argmax(S.perturbed_scores(logits, temperature, seed, position)))


_ORIG = {k: getattr(S, k) for k in ("philox4x64_10_many", "uniforms")}

MUTATIONS = [
    ("philox4x64_10", _philox_early_key_bump,
     lambda: test_philox_block_matches_numpy((0, 0, 0, 0), (0, 0))),
    ("philox4x64_10_many", _philox_many_swapped_multipliers, test_vectorised_philox_matches_numpy),
    ("uniforms", _uniforms_no_half, test_uniform_layout_and_range),
    ("uniforms", _uniforms_swapped_counter, test_uniform_layout_and_range),
    ("gumbel", _gumbel_wrong_sign, lambda: test_gumbel_max_draws_softmax(1.0)),
    ("perturbed_scores", _scores_times_t, lambda: test_gumbel_max_draws_softmax(0.7)),
    ("sample_id", _sample_id_argmin, test_limits),
]


@pytest.mark.parametrize("name,bad,pin", MUTATIONS, ids=[m[1].__name__ for m in MUTATIONS])
def test_pin_catches_planted_mistake(monkeypatch, name, bad, pin):
    monkeypatch.setattr(S, name, bad)
    with pytest.raises(AssertionError):
        pin()

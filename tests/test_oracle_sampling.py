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


# ---- filtered sampling (top-k, top-p)

def test_top_k_set_hand_examples_and_ties():
    lg = np.array([1.0, 2.0, 2.0, 0.0, 3.0])
    assert list(S.top_k_set(lg, 1)) == [4]
    assert list(S.top_k_set(lg, 2)) == [1, 4]          # tie at the boundary: lower index
    assert list(S.top_k_set(lg, 3)) == [1, 2, 4]
    assert list(S.top_k_set(lg, 0)) == list(range(5))
    assert list(S.top_k_set(lg, 9)) == list(range(5))


def test_top_p_set_hand_example_and_brute_force():
    pi = np.array([0.4, 0.25, 0.15, 0.1, 0.06, 0.04])
    lg = np.log(pi)
    assert list(S.top_p_set(lg, 1.0, 0.3)) == [0]
    assert list(S.top_p_set(lg, 1.0, 0.6)) == [0, 1]
    assert list(S.top_p_set(lg, 1.0, 0.75)) == [0, 1, 2]
    assert list(S.top_p_set(lg, 1.0, 0.97)) == [0, 1, 2, 3, 4, 5]
    assert list(S.top_p_set(lg, 1.0, 1.0)) == list(range(6))
    rng = np.random.default_rng(9)
    for _ in range(200):
        v = int(rng.integers(2, 12))
        x = rng.standard_normal(v)
        T = float(rng.uniform(0.3, 2.0))
        p = float(rng.uniform(0.05, 0.99))
        e = np.exp(x / T - np.max(x / T))
        pr = e / e.sum()
        order = sorted(range(v), key=lambda i: (-pr[i], i))
        kept, mass = [], 0.0
        for i in order:
            kept.append(i)
            mass += pr[i]
            if mass >= p:
                break
        assert list(S.top_p_set(x, T, p)) == sorted(kept)


@pytest.mark.parametrize("k,p", [(3, 1.0), (0, 0.75), (4, 0.75)])
def test_filtered_draws_follow_the_renormalised_softmax(k, p):
    pi = np.array([0.4, 0.25, 0.15, 0.1, 0.06, 0.04])
    logits = np.log(pi).astype(np.float32)
    T = 1.0
    keep = S.top_p_set(logits, T, p, among=S.top_k_set(logits, k))
    n = 40000
    sc = S.perturbed_scores(logits, T, 21, np.arange(n))
    masked = np.full_like(sc, -np.inf)
    masked[:, keep] = sc[:, keep]
    draws = np.argmax(masked, axis=1)
    assert set(np.unique(draws)) <= set(keep.tolist())
    freq = np.bincount(draws, minlength=logits.shape[0])[keep]
    q = pi[keep] / pi[keep].sum()
    chi2 = float(((freq - n * q) ** 2 / (n * q)).sum())
    assert chi2 < 30.0, (chi2, freq, n * q)
    # the per-position function agrees with the vectorised draw
    for pos in range(0, n, 4999):
        assert S.sample_id_filtered(logits, T, 21, pos, top_k=k, top_p=p) == int(draws[pos])


def test_filtered_limits():
    rng = np.random.default_rng(4)
    for pos in range(30):
        lg = rng.standard_normal(500).astype(np.float32)
        g = int(np.argmax(lg))
        assert S.sample_id_filtered(lg, 0.8, 3, pos, top_k=1) == g
        assert S.sample_id_filtered(lg, 0.8, 3, pos, top_p=1e-9) == g
        assert S.sample_id_filtered(lg, 0.0, 3, pos, top_k=5, top_p=0.5) == g
        assert S.sample_id_filtered(lg, 0.8, 3, pos, top_k=500) == S.sample_id(lg, 0.8, 3, pos)
        assert S.sample_id_filtered(lg, 0.8, 3, pos, top_p=1.0) == S.sample_id(lg, 0.8, 3, pos)


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


def _top_k_one_more(logits, k):
    lg = np.asarray(logits)
    if k <= 0 or k >= lg.shape[0]:
        return np.arange(lg.shape[0])
    return np.sort(S._order(lg)[:k + 1])


def _top_p_stops_short(logits, temperature, p, among=None):
    kept = _ORIG["top_p_set"](logits, temperature, p, among)
    return kept if kept.shape[0] == 1 or p >= 1.0 else kept[:-1]


_ORIG = {k: getattr(S, k) for k in ("philox4x64_10_many", "uniforms", "top_p_set")}

MUTATIONS = [
    ("philox4x64_10", _philox_early_key_bump,
     lambda: test_philox_block_matches_numpy((0, 0, 0, 0), (0, 0))),
    ("philox4x64_10_many", _philox_many_swapped_multipliers, test_vectorised_philox_matches_numpy),
    ("uniforms", _uniforms_no_half, test_uniform_layout_and_range),
    ("uniforms", _uniforms_swapped_counter, test_uniform_layout_and_range),
    ("gumbel", _gumbel_wrong_sign, lambda: test_gumbel_max_draws_softmax(1.0)),
    ("perturbed_scores", _scores_times_t, lambda: test_gumbel_max_draws_softmax(0.7)),
    ("sample_id", _sample_id_argmin, test_limits),
    ("top_k_set", _top_k_one_more, test_top_k_set_hand_examples_and_ties),
    ("top_p_set", _top_p_stops_short, test_top_p_set_hand_example_and_brute_force),
]


@pytest.mark.parametrize("name,bad,pin", MUTATIONS, ids=[m[1].__name__ for m in MUTATIONS])
def test_pin_catches_planted_mistake(monkeypatch, name, bad, pin):
    monkeypatch.setattr(S, name, bad)
    with pytest.raises(AssertionError):
        pin()

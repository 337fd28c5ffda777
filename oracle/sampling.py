"""CPU oracle for in-kernel token sampling (temperature sampling).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only the tests, the smoke check and the benchmark's CPU-baseline leg do.  It
shares no code with the CUDA path.

What it computes.  The pages name LM-head sampling as one of the steps the
resident decode program runs without the CPU (revietech.ru, "Kog выжимает
максимум из GPU: 3000 токенов/с", section "Что такое monokernel") but give
no sampler.  The reading taken is plain temperature sampling: the next id is
drawn from softmax(logits / T).  It is realised as the Gumbel-max
construction, which draws exactly from that distribution:

    next = argmax_i ( logits_i / T + G_i ),   G_i = -log(-log(U_i)),

with U_i independent uniforms on (0, 1) (lowest index on ties).  T -> 0
tends to greedy decoding.

Random numbers.  The uniforms cannot be passed in (the kernel draws them on
the device at every step), so both sides implement the same counter-based
generator from its published definition: Philox4x64 with 10 rounds
(Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2,
3", SC 2011).  One block of four 64-bit words per four vocabulary entries:

    words = Philox4x64-10(counter = (i // 4, position, 0, 0), key = (seed, 0))
    w     = words[i % 4]
    U_i   = ((w >> 11) + 0.5) * 2^-53           (never 0, never 1)

where `position` is the 0-based position of the token whose logits are
sampled (the step that consumes the token at position t draws with t).
"""
from __future__ import annotations

import numpy as np

# Philox4x64 constants from the published definition: the two round
# multipliers and the two Weyl-sequence key increments.
PHILOX_M0 = 0xD2E7470EE14C6C93
PHILOX_M1 = 0xCA5A826395121157
PHILOX_W0 = 0x9E3779B97F4A7C15
PHILOX_W1 = 0xBB67AE8584CAA73B
_MASK64 = (1 << 64) - 1


def philox4x64_10(counter, key):
    """One Philox4x64-10 block on Python integers: 4 counter words and 2 key
    words in, 4 64-bit words out.  Each round multiplies counter words 0 and
    2 by the two multipliers (128-bit products split into high and low
    halves), mixes the high halves with the other two counter words and the
    key, and permutes; the key advances by the Weyl increments between
    rounds."""
    c0, c1, c2, c3 = (int(v) & _MASK64 for v in counter)
    k0, k1 = (int(v) & _MASK64 for v in key)
    for r in range(10):
        if r:
            k0 = (k0 + PHILOX_W0) & _MASK64
            k1 = (k1 + PHILOX_W1) & _MASK64
        p0 = PHILOX_M0 * c0
        p1 = PHILOX_M1 * c2
        c0, c1, c2, c3 = ((p1 >> 64) ^ c1 ^ k0, p1 & _MASK64,
                          (p0 >> 64) ^ c3 ^ k1, p0 & _MASK64)
    return [c0, c1, c2, c3]


def _mulhilo(a: int, b: np.ndarray):
    """128-bit product of the constant a and each uint64 of b, as (high, low)
    uint64 arrays (schoolbook on 32-bit limbs)."""
    m32 = np.uint64(0xFFFFFFFF)
    s32 = np.uint64(32)
    a_lo, a_hi = np.uint64(a & 0xFFFFFFFF), np.uint64(a >> 32)
    b_lo, b_hi = b & m32, b >> s32
    ll = a_lo * b_lo
    lh = a_lo * b_hi
    hl = a_hi * b_lo
    hh = a_hi * b_hi
    mid = (ll >> s32) + (lh & m32) + (hl & m32)
    hi = hh + (lh >> s32) + (hl >> s32) + (mid >> s32)
    lo = (mid << s32) | (ll & m32)
    return hi, lo


def philox4x64_10_many(c0, c1, key0: int) -> np.ndarray:
    """Philox4x64-10 of the counters (c0, c1, 0, 0) under key (key0, 0),
    vectorised over c0 and c1 (broadcast against each other): returns
    uint64 [..., 4]."""
    with np.errstate(over="ignore"):
        x0, x1 = np.broadcast_arrays(np.asarray(c0, dtype=np.uint64),
                                     np.asarray(c1, dtype=np.uint64))
        x0, x1 = x0.copy(), x1.copy()
        x2 = np.zeros_like(x0)
        x3 = np.zeros_like(x0)
        k0, k1 = key0 & _MASK64, 0
        for r in range(10):
            if r:
                k0 = (k0 + PHILOX_W0) & _MASK64
                k1 = (k1 + PHILOX_W1) & _MASK64
            hi0, lo0 = _mulhilo(PHILOX_M0, x0)
            hi1, lo1 = _mulhilo(PHILOX_M1, x2)
            x0, x1, x2, x3 = (hi1 ^ x1 ^ np.uint64(k0), lo1,
                              hi0 ^ x3 ^ np.uint64(k1), lo0)
        return np.stack([x0, x1, x2, x3], axis=-1)


def uniforms(seed: int, position, n: int) -> np.ndarray:
    """U_i for vocabulary entries i = 0 .. n-1 at `position` (float64 [n]);
    `position` may be an array of positions (result [len, n])."""
    nb = (n + 3) // 4
    pos = np.asarray(position, dtype=np.uint64)
    words = philox4x64_10_many(np.arange(nb, dtype=np.uint64), pos[..., None], seed)
    words = words.reshape(pos.shape + (4 * nb,))[..., :n]
    return ((words >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53


def gumbel(u: np.ndarray) -> np.ndarray:
    """Standard Gumbel variates from uniforms on (0, 1)."""
    return -np.log(-np.log(u))


def perturbed_scores(logits: np.ndarray, temperature: float, seed: int,
                     position: int) -> np.ndarray:
    """logits / T + G (float64), the quantity whose argmax is the sample."""
    lg = np.asarray(logits, dtype=np.float64)
    return lg / float(temperature) + gumbel(uniforms(seed, position, lg.shape[0]))


def sample_id(logits: np.ndarray, temperature: float, seed: int, position: int) -> int:
    """The sampled next id: argmax of the perturbed scores, lowest index on
    ties.  temperature <= 0 means greedy (argmax of the logits)."""
    if temperature <= 0:
        return int(np.argmax(np.asarray(logits)))
    return int(np.argmax(perturbed_scores(logits, temperature, seed, position)))


def score_margin(scores: np.ndarray) -> float:
    """Top-1 minus top-2 of the perturbed scores."""
    s = np.sort(np.asarray(scores, dtype=np.float64))
    return float(s[-1] - s[-2]) if s.shape[0] > 1 else float("inf")


# ---- filtered sampling (top-k, top-p).  The kernel does not draw these
# yet; they are defined here first so that its draws can be checked.
#
# top-k keeps the k largest logits (ties broken by the lower index); top-p
# (nucleus) keeps, of the remaining entries ordered by probability under
# softmax(logits / T) (ties by the lower index), the shortest prefix whose
# probability mass reaches p, renormalised over the kept set.  The draw is
# the Gumbel-max one above restricted to the kept set, with the same
# noise, so an entry's score does not depend on the filter.

def _order(values: np.ndarray) -> np.ndarray:
    """Indices by value, largest first, ties by the lower index."""
    v = np.asarray(values, dtype=np.float64)
    return np.lexsort((np.arange(v.shape[0]), -v))


def top_k_set(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits (all of them for k <= 0 or k >= V)."""
    lg = np.asarray(logits)
    if k <= 0 or k >= lg.shape[0]:
        return np.arange(lg.shape[0])
    return np.sort(_order(lg)[:k])


def top_p_set(logits: np.ndarray, temperature: float, p: float,
              among: np.ndarray = None) -> np.ndarray:
    """The nucleus: of the entries `among` (default all), ordered by
    probability under softmax(logits / T) restricted to them, the shortest
    prefix whose mass reaches p (at least one entry; all for p >= 1)."""
    lg = np.asarray(logits, dtype=np.float64)
    idx = np.arange(lg.shape[0]) if among is None else np.asarray(among)
    if p >= 1.0:
        return np.sort(idx)
    z = lg[idx] / float(temperature)
    pr = np.exp(z - z.max())
    pr /= pr.sum()
    o = _order(pr)
    mass = np.cumsum(pr[o])
    n = int(np.searchsorted(mass, p, side="left")) + 1
    return np.sort(idx[o[:min(n, idx.shape[0])]])


def sample_id_filtered(logits: np.ndarray, temperature: float, seed: int, position: int,
                       top_k: int = 0, top_p: float = 1.0) -> int:
    """Draw restricted to top-k, then top-p of what top-k kept.  T <= 0 is
    greedy (the argmax lies in every non-empty kept set)."""
    if temperature <= 0:
        return int(np.argmax(np.asarray(logits)))
    keep = top_k_set(logits, top_k)
    keep = top_p_set(logits, temperature, top_p, among=keep)
    sc = perturbed_scores(logits, temperature, seed, position)
    return int(keep[np.argmax(sc[keep])])

"""In-kernel temperature sampling and the EOS id set, through the C ABI,
against the sampling oracle (`oracle.sampling`) on the oracle model.

Bar, per teacher-forced step (rows of prefill + forced decode):
  * logits within the parity bar (max |dlogit| <= 1e-2 * max |oracle|);
  * the GPU's id is the argmax of its OWN logits / T plus the oracle's
    Gumbel noise wherever that score's top-2 margin exceeds 1e-3: this
    checks the kernel's Philox words, their map to (0, 1), the Gumbel
    transform and the argmax exactly, independent of logit rounding;
  * the GPU's id equals the oracle's draw (oracle logits / T + noise)
    wherever the oracle's score margin exceeds what the allowed logit error
    can move, 2 * 1e-2 * max |oracle logit| / T.
"""
import numpy as np
import pytest

import synth
from oracle import OracleModel
from oracle import sampling as S
from parity import LOGIT_RTOL, device_model

pytestmark = pytest.mark.gpu

OWN_MARGIN = 1e-3


@pytest.fixture(scope="module")
def tiny():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from persistent_sm_decode_monokernel_b200 import build
    build.build()
    w = synth.WORKLOADS["tiny-l2-d256"]
    m = synth.make_model(w.shape, seed=0)
    return w, m, device_model(m), synth.make_prompt(w.shape.vocab, w.prompt_len, seed=0)


def _session(w, dev, max_seq, eos=-1):
    from persistent_sm_decode_monokernel_b200 import Session
    return Session(w.shape, dev, max_seq=max_seq, eos_id=eos)


def _forced_sampled(w, m, dev, prompt, n, T, seed):
    """(gpu logits [n+1, V], gpu ids [n+1], oracle logits, positions)."""
    forced = synth.make_forced_ids(w.shape.vocab, n, seed=5)
    s = _session(w, dev, len(prompt) + n)
    s.set_sampling(T, seed)
    cap0 = s.capture_logits(1)
    g0 = s.prefill(prompt)
    l0 = cap0.cpu().numpy().copy()
    cap = s.capture_logits(n)
    picks = s.decode_forced(forced)
    lg = np.concatenate([l0, cap.cpu().numpy()])
    s.close()
    seq = np.concatenate([prompt, forced])
    P = len(prompt)
    ref = OracleModel(m, dtype=np.float32).forward(seq, logits_rows=range(P - 1, len(seq)))
    positions = np.arange(P - 1, len(seq))
    return lg, np.concatenate([[g0], picks]).astype(np.int64), ref, positions


def _check_rows(lg, ids, ref, positions, T, seed):
    V = lg.shape[1]
    own_checked = ref_checked = 0
    for i, pos in enumerate(positions):
        r = ref[i].astype(np.float64)
        g = lg[i].astype(np.float64)
        scale = np.max(np.abs(r))
        assert np.max(np.abs(g - r)) <= LOGIT_RTOL * scale, f"row {i}: logits off"
        noise = S.gumbel(S.uniforms(seed, int(pos), V))
        own = g / T + noise
        if S.score_margin(own) > OWN_MARGIN:
            own_checked += 1
            assert int(ids[i]) == int(np.argmax(own)), (
                f"row {i}: gpu id {ids[i]} != argmax of its own noisy scores {np.argmax(own)}")
        sc = r / T + noise
        if S.score_margin(sc) > 2 * LOGIT_RTOL * scale / T:
            ref_checked += 1
            assert int(ids[i]) == int(np.argmax(sc)), (
                f"row {i}: gpu id {ids[i]} != oracle draw {np.argmax(sc)}")
    return own_checked, ref_checked


@pytest.mark.parametrize("T,seed", [(0.7, 1234), (1.5, 99), (1.0, (1 << 64) - 3)])
def test_sampled_ids_match_oracle_teacher_forced(tiny, T, seed):
    w, m, dev, prompt = tiny
    lg, ids, ref, positions = _forced_sampled(w, m, dev, prompt, 32, T, seed)
    own, refc = _check_rows(lg, ids, ref, positions, T, seed)
    assert own >= 30 and refc >= 20, (own, refc)
    # sampling is active: the picks are not all the greedy ones
    assert np.sum(ids != np.argmax(lg, axis=1)) > 5


def test_huge_temperature_draws_follow_the_generator_alone(tiny):
    w, m, dev, prompt = tiny
    lg, ids, ref, positions = _forced_sampled(w, m, dev, prompt, 24, 1e6, 7)
    for i, pos in enumerate(positions):
        u = S.uniforms(7, int(pos), w.shape.vocab)
        top2 = np.sort(S.gumbel(u))[-2:]
        if top2[1] - top2[0] > 1e-4:
            assert int(ids[i]) == int(np.argmax(u)), f"row {i}"


def test_free_running_sampled_decode_matches_oracle(tiny):
    w, m, dev, prompt = tiny
    # with this seed every draw of the oracle's own run has a score margin
    # at least 3.5 times what the allowed logit error can move, so the whole
    # run must agree
    T, seed, n = 1.0, 4244, 24
    s = _session(w, dev, len(prompt) + n + 1)
    s.set_sampling(T, seed)
    cap0 = s.capture_logits(1)
    g0 = s.prefill(prompt)
    l0 = cap0.cpu().numpy().copy()
    cap = s.capture_logits(n)
    out = list(s.decode(n))
    lg = np.concatenate([l0, cap.cpu().numpy()])
    s.close()
    gpu = [g0] + out
    om = OracleModel(m, dtype=np.float32)
    st = om.new_state()
    logits = om.prefill(st, prompt)
    P = len(prompt)
    compared = 0
    for i in range(n + 1):
        pos = P - 1 + i
        r = logits.astype(np.float64)
        scale = np.max(np.abs(r))
        assert np.max(np.abs(lg[i].astype(np.float64) - r)) <= LOGIT_RTOL * scale
        sc = r / T + S.gumbel(S.uniforms(seed, pos, w.shape.vocab))
        want = int(np.argmax(sc))
        if gpu[i] != want:
            # a legitimate flip only where the logit error could move the draw
            assert S.score_margin(sc) <= 2 * LOGIT_RTOL * scale / T, f"step {i}"
            break
        compared += 1
        if i < n:
            logits = om.decode_step(st, want)
    assert compared == n + 1


def test_seed_reproducible_rewind_and_temperature_zero(tiny):
    w, m, dev, prompt = tiny
    s = _session(w, dev, 64)
    s.prefill(prompt)
    greedy = list(s.decode(20))
    s.set_sampling(1.0, 11)
    s.rewind(len(prompt))
    a = list(s.decode(20))
    s.rewind(len(prompt))
    b = list(s.decode(20))
    assert a == b                       # same seed, same positions: same draws
    s.set_sampling(1.0, 12)
    s.rewind(len(prompt))
    c = list(s.decode(20))
    assert c != a
    assert a != greedy
    s.set_sampling(0.0, 11)             # back to greedy
    s.rewind(len(prompt))
    assert list(s.decode(20)) == greedy
    for tiny_t in (1e-30, 1e-6):        # the T -> 0 limit is the greedy pick
        s.set_sampling(tiny_t, 11)
        s.rewind(len(prompt))
        assert list(s.decode(20)) == greedy
    # the first id of a sampled prefill is drawn too (position P - 1)
    s.set_sampling(1e6, 3)
    g = s.prefill(prompt)
    assert g == int(np.argmax(S.uniforms(3, len(prompt) - 1, w.shape.vocab)))
    s.close()


def test_eos_id_set(tiny):
    from persistent_sm_decode_monokernel_b200 import KieError, _kie
    w, m, dev, prompt = tiny
    s = _session(w, dev, 64)
    s.prefill(prompt)
    ids = list(s.decode(20))
    k = 7
    stop = ids[k]
    first = ids.index(stop)
    unused = next(v for v in range(w.shape.vocab) if v not in ids)
    s.set_eos_ids([unused, stop])
    s.rewind(len(prompt))
    out = list(s.decode(20))
    assert out == ids[:first + 1]
    assert s.stats()["pos"] == len(prompt) + first + 1
    s.set_eos_ids([])                   # back to the descriptor's (none)
    s.rewind(len(prompt))
    assert list(s.decode(20)) == ids
    for bad in ([w.shape.vocab], [-1], list(range(_kie.KIE_MAX_EOS_IDS + 1))):
        with pytest.raises(KieError) as e:
            s.set_eos_ids(bad)
        assert e.value.status == _kie.KIE_ERR_INVALID_ARG
    for bad_t in (-1.0, float("inf"), float("nan")):
        with pytest.raises(KieError) as e:
            s.set_sampling(bad_t, 0)
        assert e.value.status == _kie.KIE_ERR_INVALID_ARG
    s.close()

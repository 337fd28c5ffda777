"""In-kernel top-k / top-p sampling through the C ABI, against the sampling
oracle's filtered draw (`oracle.sampling.sample_id_filtered`: the top_k
largest logits, ties by the lower id, then the nucleus of those under
softmax(logits / T), then the Gumbel-max draw over the kept ids).

Bar, per teacher-forced step:
  * logits within the parity bar;
  * the GPU's id equals the oracle's filter and draw applied to the GPU's
    OWN logits with the oracle's noise, wherever that is decided by more
    than rounding: the top-k set is then exact (it is the same order on the
    same fp32 values), the top-p cut is skipped when a probability-mass
    prefix lies within 1e-9 of top_p (fp64 sums in another order), and the
    draw when its score margin among the kept ids is below 1e-3;
  * the GPU's id equals the oracle's draw on the oracle's own logits
    wherever both logit vectors keep the same set and the oracle's score
    margin in it exceeds what the allowed logit error can move.
"""
import numpy as np
import pytest

import synth
from oracle import OracleModel
from oracle import sampling as S
from parity import LOGIT_RTOL, device_model

pytestmark = pytest.mark.gpu

OWN_MARGIN = 1e-3
MASS_EPS = 1e-9


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from persistent_sm_decode_monokernel_b200 import build
    build.build()
    return torch


@pytest.fixture(scope="module")
def tiny(torch_cuda):
    w = synth.WORKLOADS["tiny-l2-d256"]
    m = synth.make_model(w.shape, seed=0)
    return w, m, device_model(m), synth.make_prompt(w.shape.vocab, w.prompt_len, seed=0)


def _forced(w, m, dev, prompt, n, T, seed, k, p, forced_seed=5):
    from persistent_sm_decode_monokernel_b200 import Session
    forced = synth.make_forced_ids(w.shape.vocab, n, seed=forced_seed)
    s = Session(w.shape, dev, max_seq=len(prompt) + n)
    s.set_sampling(T, seed, top_k=k, top_p=p)
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
    return lg, np.concatenate([[g0], picks]).astype(np.int64), ref, np.arange(P - 1, len(seq))


def _kept(logits, T, k, p):
    keep = S.top_k_set(logits, k)
    return S.top_p_set(logits, T, p, among=keep)


def _cut_is_clear(logits, T, k, p):
    """No probability-mass prefix of the top-k set within MASS_EPS of p."""
    if p >= 1.0:
        return True
    idx = S.top_k_set(logits, k)
    z = np.asarray(logits, dtype=np.float64)[idx] / T
    pr = np.exp(z - z.max())
    pr /= pr.sum()
    mass = np.cumsum(pr[S._order(pr)])
    return bool(np.all(np.abs(mass - p) > MASS_EPS))


def _margin_in(scores, keep):
    return S.score_margin(scores[keep]) if len(keep) > 1 else float("inf")


def _check(lg, ids, ref, positions, T, seed, k, p, against_oracle=True):
    """against_oracle=False checks the selection on the GPU's own logits only
    (for models outside the logit bar's scope)."""
    V = lg.shape[1]
    own_checked = ref_checked = 0
    for i, pos in enumerate(positions):
        r = ref[i].astype(np.float64) if against_oracle else None
        g = lg[i].astype(np.float64)
        if against_oracle:
            scale = np.max(np.abs(r))
            assert np.max(np.abs(g - r)) <= LOGIT_RTOL * scale, f"row {i}: logits off"
        noise = S.gumbel(S.uniforms(seed, int(pos), V))
        keep_g = _kept(g, T, k, p)
        assert int(ids[i]) in set(keep_g.tolist()) or not _cut_is_clear(g, T, k, p), (
            f"row {i}: gpu id {ids[i]} outside the kept set of its own logits")
        own = g / T + noise
        if _cut_is_clear(g, T, k, p) and _margin_in(own, keep_g) > OWN_MARGIN:
            own_checked += 1
            want = int(keep_g[np.argmax(own[keep_g])])
            assert int(ids[i]) == want, f"row {i}: gpu id {ids[i]} != own-logit draw {want}"
        if not against_oracle:
            continue
        keep_r = _kept(r, T, k, p)
        sc = r / T + noise
        if (np.array_equal(keep_r, keep_g) and _cut_is_clear(r, T, k, p)
                and _margin_in(sc, keep_r) > 2 * LOGIT_RTOL * scale / T):
            ref_checked += 1
            want = S.sample_id_filtered(r, T, seed, int(pos), top_k=k, top_p=p)
            assert int(ids[i]) == want, f"row {i}: gpu id {ids[i]} != oracle draw {want}"
    return own_checked, ref_checked


@pytest.mark.parametrize("T,seed,k,p", [
    (1.0, 5, 1, 1.0),        # top-1: the greedy pick
    (1.0, 7, 5, 1.0),
    (0.8, 9, 40, 1.0),
    (1.0, 11, 64, 0.9),
    (1.5, 13, 20, 0.5),
    (1.0, 17, 64, 0.3),
])
def test_filtered_draws_match_oracle_teacher_forced(tiny, T, seed, k, p):
    w, m, dev, prompt = tiny
    lg, ids, ref, positions = _forced(w, m, dev, prompt, 32, T, seed, k, p)
    own, refc = _check(lg, ids, ref, positions, T, seed, k, p)
    assert own >= 28 and refc >= 20, (own, refc)
    if k == 1:
        assert np.array_equal(ids, np.argmax(lg, axis=1))


def test_many_candidates_from_one_cta_and_ties(tiny):
    # 64 rows of the LM head share one row scaled up, 64 more its negative:
    # at almost every step one group holds the 64 largest (near-tied)
    # logits, so the global top-40 lies in a few CTAs' ~14 rows each -- more
    # than the 8 entries of a list every CTA copies -- and the tie rule
    # decides order.  The 200-fold rows also scale the fp16 rounding of the
    # GEMV input 200-fold, beyond the logit bar (which is relative to the
    # step's largest logit), so the draw is checked on the GPU's own logits.
    w, m, _, prompt = tiny
    lm = m.tensors["lm_head"].astype(np.float32).copy()
    a = lm[1000] * 200.0
    lm[0:64] = a
    lm[64:128] = -a
    over = synth.make_model(w.shape, seed=0, overrides={"lm_head": lm.astype(np.float16)})
    dev = device_model(over)
    lg, ids, ref, positions = _forced(w, over, dev, prompt, 16, 1.0, 23, 40, 1.0)
    own, _ = _check(lg, ids, ref, positions, 1.0, 23, 40, 1.0, against_oracle=False)
    assert own >= 14, own
    # on most steps the planted group holds the whole top-40
    grouped = sum(int(np.all(S.top_k_set(row, 40) < 128)) for row in lg)
    assert grouped >= 12, grouped


def test_filter_arguments(tiny):
    from persistent_sm_decode_monokernel_b200 import KieError, Session, _kie
    w, m, dev, prompt = tiny
    s = Session(w.shape, dev, max_seq=64)
    s.prefill(prompt)
    greedy = list(s.decode(8))
    for k, p, st in [(-1, 1.0, _kie.KIE_ERR_INVALID_ARG), (_kie.KIE_MAX_TOP_K + 1, 1.0,
                                                           _kie.KIE_ERR_INVALID_ARG),
                     (5, 0.0, _kie.KIE_ERR_INVALID_ARG), (5, 1.5, _kie.KIE_ERR_INVALID_ARG),
                     (0, 0.9, _kie.KIE_ERR_UNSUPPORTED)]:
        with pytest.raises(KieError) as e:
            s.set_sampling(1.0, 3, top_k=k, top_p=p)
        assert e.value.status == st, (k, p)
    # a filter leaves greedy decoding unchanged
    s.set_sampling(0.0, 3, top_k=5, top_p=0.5)
    s.rewind(len(prompt))
    assert list(s.decode(8)) == greedy
    s.close()

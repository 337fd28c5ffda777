"""Parity of the CUDA decode path (through the C ABI) against the CPU oracle.

Bar (per compared step): max |logit_gpu - logit_oracle| <= 1e-2 * max |logit_oracle|,
and the greedy id equal to the oracle's argmax wherever the oracle's top-1 /
top-2 margin exceeds 2e-2.  The GPU keeps K/V in fp16 and activations in
fp32; the oracle computes in fp32 with an fp32 cache.
"""
import numpy as np
import pytest

import synth
from oracle import OracleModel
from parity import compare_free_running, compare_steps, device_model

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from persistent_sm_decode_monokernel_b200 import build
    build.build()
    return torch


def _session(shape, dev, max_seq, eos=-1):
    from persistent_sm_decode_monokernel_b200 import Session
    return Session(shape, dev, max_seq=max_seq, eos_id=eos)


def _run_free(sess, prompt, n_steps):
    cap0 = sess.capture_logits(1)
    g0 = sess.prefill(prompt)
    l0 = cap0.cpu().numpy().copy()
    cap = sess.capture_logits(max(n_steps, 1))
    ids = sess.decode(n_steps)
    lg = cap.cpu().numpy()[:len(ids)]
    sess.capture_off()
    return [g0] + [int(x) for x in ids], np.concatenate([l0, lg])


def _run_forced(sess, prompt, forced):
    cap0 = sess.capture_logits(1)
    g0 = sess.prefill(prompt)
    l0 = cap0.cpu().numpy().copy()
    cap = sess.capture_logits(len(forced))
    picks = sess.decode_forced(forced)
    lg = cap.cpu().numpy()
    sess.capture_off()
    return np.concatenate([[g0], picks]), np.concatenate([l0, lg])


SMALL = ["tiny-l2-d256", "l16-d1024"]


@pytest.mark.parametrize("name", SMALL)
def test_free_running_greedy_matches_oracle(torch_cuda, name):
    w = synth.WORKLOADS[name]
    m = synth.make_model(w.shape, seed=w.seed)
    prompt = synth.make_prompt(w.shape.vocab, w.prompt_len, seed=w.seed)
    sess = _session(w.shape, device_model(m), w.max_seq)
    gpu_ids, gpu_lg = _run_free(sess, prompt, w.decode_steps)
    sess.close()
    or_ids, or_lg = OracleModel(m, dtype=np.float32).greedy(prompt, w.decode_steps,
                                                             batched_prefill=True)
    rep = compare_free_running(gpu_ids, gpu_lg, or_ids, or_lg)
    assert rep.compared >= 1
    print(f"{name}: compared {rep.compared} steps, worst rel {rep.worst_rel:.2e}, "
          f"ids checked {rep.id_checked}, divergence at {rep.first_divergence}")


@pytest.mark.parametrize("name", SMALL)
def test_teacher_forced_logits_match_oracle(torch_cuda, name):
    w = synth.WORKLOADS[name]
    m = synth.make_model(w.shape, seed=w.seed)
    prompt = synth.make_prompt(w.shape.vocab, w.prompt_len, seed=w.seed)
    forced = synth.make_forced_ids(w.shape.vocab, w.decode_steps, seed=w.seed)
    sess = _session(w.shape, device_model(m), w.max_seq)
    picks, gpu_lg = _run_forced(sess, prompt, forced)
    sess.close()
    seq = np.concatenate([prompt, forced])
    om = OracleModel(m, dtype=np.float32)
    ref = om.forward(seq, logits_rows=range(w.prompt_len - 1, len(seq)))
    rep = compare_steps(gpu_lg, picks, ref)
    assert rep.id_checked > 0.5 * rep.compared
    print(f"{name}: {rep.compared} steps, worst rel {rep.worst_rel:.2e}")

"""Parity at the benchmark's full sizes, in the launch configuration the
benchmark times (prefill of the whole prompt in one launch, then all
decode steps of the request in one launch).

Every decode step's logits are compared with the oracle's on a seeded
teacher-forcing stream (the GPU is fed the same ids the oracle is), and the
first free-running greedy steps are compared with the oracle's own greedy
decode.  The oracle runs in fp32 on the host cores; the 8k-context and 8B
cases take a minute or two of CPU time each.
"""
import numpy as np
import pytest

import synth
from oracle import OracleModel
from parity import compare_free_running, compare_steps, device_model

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = ["l28-d2560", "l28-d2560-ctx8k", "l32-d4096"]


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from persistent_sm_decode_monokernel_b200 import build
    build.build()
    return torch


@pytest.mark.parametrize("name", FULL)
def test_full_size_forced_and_greedy(torch_cuda, name):
    from persistent_sm_decode_monokernel_b200 import Session
    w = synth.WORKLOADS[name]
    m = synth.make_model(w.shape, seed=w.seed)
    prompt = synth.make_prompt(w.shape.vocab, w.prompt_len, seed=w.seed)
    forced = synth.make_forced_ids(w.shape.vocab, w.decode_steps, seed=w.seed)
    dev = device_model(m)
    s = Session(w.shape, dev, max_seq=w.max_seq)
    cap0 = s.capture_logits(1)
    g0 = s.prefill(prompt)
    l0 = cap0.cpu().numpy().copy()
    s.capture_off()
    n_free = 4
    cap = s.capture_logits(n_free)
    free = [g0] + [int(x) for x in s.decode(n_free)]
    lf = np.concatenate([l0, cap.cpu().numpy()])
    s.rewind(w.prompt_len)
    cap = s.capture_logits(w.decode_steps)
    picks = s.decode_forced(forced)
    lg = np.concatenate([l0, cap.cpu().numpy()])
    s.close()
    del dev, cap, cap0
    torch_cuda.cuda.empty_cache()

    om = OracleModel(m, dtype=np.float32)
    seq = np.concatenate([prompt, forced])
    ref = om.forward(seq, logits_rows=range(w.prompt_len - 1, len(seq)))
    rep = compare_steps(lg, np.concatenate([[g0], picks]), ref)
    assert rep.compared == w.decode_steps + 1
    assert rep.id_checked > 0.5 * rep.compared
    or_ids, or_lg = om.greedy(prompt, n_free, batched_prefill=True)
    rep2 = compare_free_running(free, lf, or_ids, or_lg)
    print(f"{name}: forced {rep.compared} steps worst rel {rep.worst_rel:.2e}; "
          f"greedy {rep2.compared} steps (divergence {rep2.first_divergence})")

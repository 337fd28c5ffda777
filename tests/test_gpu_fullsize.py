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


def test_full_size_sampled_draws(torch_cuda):
    # the draw reads the LM-head slices of every CTA (~340 rows each at the
    # 50304-word vocabulary): 64 teacher-forced steps of the 2.2B model,
    # temperature sampling alone and restricted to top-40 / top-0.9, against
    # the sampling oracle (bar of test_gpu_sampling_filtered)
    import dataclasses
    from persistent_sm_decode_monokernel_b200 import Session
    from test_gpu_sampling_filtered import _check
    w = dataclasses.replace(synth.WORKLOADS["l28-d2560"], decode_steps=64)
    m = synth.make_model(w.shape, seed=w.seed)
    prompt = synth.make_prompt(w.shape.vocab, w.prompt_len, seed=w.seed)
    forced = synth.make_forced_ids(w.shape.vocab, w.decode_steps, seed=w.seed)
    dev = device_model(m)
    runs = []
    for T, seed, k, p in [(1.0, 3, 0, 1.0), (1.0, 5, 40, 0.9)]:
        s = Session(w.shape, dev, max_seq=w.max_seq)
        s.set_sampling(T, seed, top_k=k, top_p=p)
        cap0 = s.capture_logits(1)
        g0 = s.prefill(prompt)
        l0 = cap0.cpu().numpy().copy()
        cap = s.capture_logits(w.decode_steps)
        picks = s.decode_forced(forced)
        runs.append((T, seed, k, p, np.concatenate([l0, cap.cpu().numpy()]),
                     np.concatenate([[g0], picks]).astype(np.int64)))
        s.close()
    del dev
    torch_cuda.cuda.empty_cache()
    seq = np.concatenate([prompt, forced])
    P = w.prompt_len
    ref = OracleModel(m, dtype=np.float32).forward(seq, logits_rows=range(P - 1, len(seq)))
    positions = np.arange(P - 1, len(seq))
    for T, seed, k, p, lg, ids in runs:
        own, refc = _check(lg, ids, ref, positions, T, seed, k, p)
        assert own >= 55 and refc >= 30, (T, k, p, own, refc)
        print(f"sampled T={T} top_k={k} top_p={p}: own-logit draws checked {own}, "
              f"oracle draws checked {refc} of {len(ids)}")

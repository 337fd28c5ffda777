"""FP8 E4M3 weight stream (KIE_OPT_WEIGHT_FP8) through the C ABI, against the
FP8 oracle (`oracle.fp8`).

  * the quantisation is byte and bit work, so it must be exact: codes and
    fp32 row scales from kie_quantize_e4m3 (the rule the packed stream uses)
    equal oracle.fp8.quantize_rows on matrices with zero rows, subnormal
    codes, ties and the largest fp16 values;
  * decode with FP8 weights is compared with the oracle run on the
    dequantised model (every matrix replaced by s_r * value(code)), at the
    parity bar of the fp16 path: teacher-forced logits within 1e-2 of
    max |logit| at every step, greedy ids equal where the oracle's top-2
    margin exceeds 2e-2, and each pick the argmax of the GPU's own logits.
"""
import dataclasses

import numpy as np
import pytest

import synth
from oracle import OracleModel
from oracle import fp8 as F
from parity import compare_steps, device_model

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from persistent_sm_decode_monokernel_b200 import build
    build.build()
    return torch


def _quantize_gpu(torch, W16):
    from persistent_sm_decode_monokernel_b200 import _kie
    W = torch.from_numpy(W16).cuda()
    N, K = W16.shape
    codes = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    scales = torch.empty(N, dtype=torch.float32, device="cuda")
    _kie.kie_quantize_e4m3(W, codes, scales, stream=torch.cuda.current_stream().cuda_stream)
    return codes.cpu().numpy(), scales.cpu().numpy()


def test_quantize_codes_and_scales_bit_exact(torch_cuda):
    rng = np.random.default_rng(0)
    cases = []
    W = (rng.standard_normal((300, 512)) * 0.02).astype(np.float16)
    W[5] = 0                                           # zero row: scale 1, codes 0
    W[6, :] = np.float16(1e-7)                         # fp16 subnormals, one value
    W[7, ::3] = np.float16(65504)                      # largest fp16 magnitudes
    W[7, 1::3] = np.float16(-65504)
    cases.append(W)
    # rows whose quotients fall exactly on E4M3 midpoints (ties to even)
    vals = F.e4m3_value(np.arange(127, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2)
    T = np.zeros((4, 256), dtype=np.float32)
    T[:, 0] = 448.0                                    # scale exactly 1
    T[:, 1:1 + 126] = mids[None, :] * np.array([1, -1, 1, -1])[:, None]
    cases.append(T.astype(np.float16))
    cases.append((rng.standard_normal((64, 6912)) * rng.uniform(0.001, 3, (64, 1))).astype(np.float16))
    for W16 in cases:
        codes, scales = _quantize_gpu(torch_cuda, W16)
        want_c, want_s = F.quantize_rows(W16)
        np.testing.assert_array_equal(scales.view(np.uint32), want_s.view(np.uint32))
        np.testing.assert_array_equal(codes, want_c)


def _fp8_forced(torch, w, n_steps):
    from persistent_sm_decode_monokernel_b200 import Session
    m = synth.make_model(w.shape, seed=w.seed)
    prompt = synth.make_prompt(w.shape.vocab, w.prompt_len, seed=w.seed)
    forced = synth.make_forced_ids(w.shape.vocab, n_steps, seed=w.seed)
    dev = device_model(m)
    s = Session(w.shape, dev, max_seq=w.prompt_len + n_steps, weight_format="fp8",
                keep_matrices=False)
    del dev
    cap0 = s.capture_logits(1)
    g0 = s.prefill(prompt)
    l0 = cap0.cpu().numpy().copy()
    cap = s.capture_logits(n_steps)
    picks = s.decode_forced(forced)
    lg = np.concatenate([l0, cap.cpu().numpy()])
    s.close()
    torch.cuda.empty_cache()
    q, _ = F.fp8_model(m, dtype=np.float32)
    seq = np.concatenate([prompt, forced])
    ref = OracleModel(q, dtype=np.float32).forward(seq, logits_rows=range(w.prompt_len - 1, len(seq)))
    return compare_steps(lg, np.concatenate([[g0], picks]), ref), lg, ref, m, seq


@pytest.mark.parametrize("name,steps", [("tiny-l2-d256", 32), ("l16-d1024", 48)])
def test_fp8_decode_matches_fp8_oracle(torch_cuda, name, steps):
    rep, lg, ref, m, seq = _fp8_forced(torch_cuda, synth.WORKLOADS[name], steps)
    assert rep.compared == steps + 1
    assert rep.id_checked > 0.5 * rep.compared
    # the FP8 model is a different model: its logits move away from the
    # fp16 model's by far more than the parity bar
    P = synth.WORKLOADS[name].prompt_len
    r16 = OracleModel(m, dtype=np.float32).forward(seq, logits_rows=range(P - 1, len(seq)))
    assert np.max(np.abs(r16 - ref)) > 3e-2 * np.max(np.abs(ref))


@pytest.mark.slow
def test_fp8_decode_full_size_l28(torch_cuda):
    w = dataclasses.replace(synth.WORKLOADS["l28-d2560"], decode_steps=32)
    rep, *_ = _fp8_forced(torch_cuda, w, 32)
    assert rep.compared == 33
    print(f"l28-d2560 fp8: forced 33 steps worst rel {rep.worst_rel:.2e}, ids checked "
          f"{rep.id_checked}")


def test_fp8_option_switches_back(torch_cuda):
    from persistent_sm_decode_monokernel_b200 import Session, _kie
    w = synth.WORKLOADS["tiny-l2-d256"]
    m = synth.make_model(w.shape, seed=0)
    prompt = synth.make_prompt(w.shape.vocab, w.prompt_len, seed=0)
    s = Session(w.shape, device_model(m), max_seq=64)
    s.prefill(prompt)
    a = list(s.decode(16))
    s.set_option(_kie.KIE_OPT_WEIGHT_FP8, 1)
    s.prefill(prompt)
    b = list(s.decode(16))
    s.set_option(_kie.KIE_OPT_WEIGHT_FP8, 0)
    s.prefill(prompt)
    assert list(s.decode(16)) == a
    assert b != a
    s.close()

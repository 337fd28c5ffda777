"""Batched prefill (tcgen05 tensor-core GEMMs over the prompt; on by default)
through the C ABI, against the oracle's batched prefill.

Every prefilled K and V row of every layer (fp16 in the cache) is compared
with the oracle's fp32 K (after RoPE) and V of the same position: per layer
and matrix, max |gpu - oracle| <= 1e-2 * max |oracle|, the logit bar applied
to the cache (the GPU rounds GEMM inputs and the cache to fp16, the oracle
keeps fp32; the fp16 rounding of the cache alone is 2^-11 relative).  The
last position's logits (one decode step after the batched positions) meet
the logit bar against the oracle, and its pick is the oracle's argmax where
the top-2 margin exceeds 2e-2.  The batched path also agrees with the
position-by-position prefill of the decode kernel on the same bar.
"""
import numpy as np
import pytest

import synth
from oracle import OracleModel, top2_margin
from parity import LOGIT_RTOL, MARGIN, device_model

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from persistent_sm_decode_monokernel_b200 import build
    build.build()
    return torch


def _cache(s, shape, P):
    """GPU K and V of positions 0..P-1: [L, 2, KV, P, hd] fp64."""
    kv = s.kv.view(shape.n_layers, 2, shape.n_kv_heads, -1, shape.head_dim + 8)
    return kv[:, :, :, :P, :shape.head_dim].double().cpu().numpy()


def _prefill(torch, shape, dev, prompt, batched):
    from persistent_sm_decode_monokernel_b200 import Session, _kie
    s = Session(shape, dev, max_seq=len(prompt) + 1)
    s.set_option(_kie.KIE_OPT_BATCHED_PREFILL, 1 if batched else 0)
    cap = s.capture_logits(1)
    g0 = s.prefill(prompt)
    st = s.stats()
    assert st["last_prefill_batched"] == (1 if batched else 0)
    lg = cap.cpu().numpy()[0].astype(np.float64)
    kv = _cache(s, shape, len(prompt))
    s.close()
    return g0, lg, kv, st["last_prefill_ms"]


def _check_cache(kv, ref_kv, what):
    for l in range(kv.shape[0]):
        for m in range(2):
            ref = ref_kv[l, m]
            err = np.max(np.abs(kv[l, m] - ref))
            assert err <= LOGIT_RTOL * np.max(np.abs(ref)), (what, l, "KV"[m], err)


def _oracle(m, prompt):
    st, lg = OracleModel(m, dtype=np.float32).prefill_batched(prompt)
    L = len(st.k)
    # [L, 2, KV, P, hd]
    ref = np.stack([np.stack([np.stack(st.k[l], axis=1), np.stack(st.v[l], axis=1)])
                    for l in range(L)]).astype(np.float64)
    return ref, lg.astype(np.float64)


def _check_all(torch, w, m, P):
    prompt = synth.make_prompt(w.shape.vocab, P, seed=w.seed)
    dev = device_model(m)
    g0, lg, kv, ms = _prefill(torch, w.shape, dev, prompt, True)
    del dev
    torch.cuda.empty_cache()
    ref_kv, ref_lg = _oracle(m, prompt)
    _check_cache(kv, ref_kv, "batched")
    scale = np.max(np.abs(ref_lg))
    assert np.max(np.abs(lg - ref_lg)) <= LOGIT_RTOL * scale
    assert g0 == int(np.argmax(lg))
    if top2_margin(ref_lg) > MARGIN:
        assert g0 == int(np.argmax(ref_lg))
    return ms


@pytest.mark.parametrize("P", [2, 16, 129, 300])
def test_batched_prefill_matches_oracle_tiny(torch_cuda, P):
    w = synth.WORKLOADS["tiny-l2-d256"]
    _check_all(torch_cuda, w, synth.make_model(w.shape, seed=0), P)


def test_batched_prefill_matches_oracle_l16(torch_cuda):
    w = synth.WORKLOADS["l16-d1024"]
    _check_all(torch_cuda, w, synth.make_model(w.shape, seed=0), 128)


def test_batched_equals_position_by_position_prefill(torch_cuda):
    w = synth.WORKLOADS["l16-d1024"]
    m = synth.make_model(w.shape, seed=0)
    prompt = synth.make_prompt(w.shape.vocab, 200, seed=3)
    dev = device_model(m)
    ga, la, kva, _ = _prefill(torch_cuda, w.shape, dev, prompt, True)
    gb, lb, kvb, _ = _prefill(torch_cuda, w.shape, dev, prompt, False)
    _check_cache(kva, kvb, "batched vs sequential")
    assert np.max(np.abs(la - lb)) <= LOGIT_RTOL * np.max(np.abs(lb))
    if top2_margin(lb) > MARGIN:
        assert ga == gb


@pytest.mark.slow
@pytest.mark.parametrize("name", ["l28-d2560", "l28-d2560-ctx8k"])
def test_batched_prefill_full_size(torch_cuda, name):
    w = synth.WORKLOADS[name]
    ms = _check_all(torch_cuda, w, synth.make_model(w.shape, seed=w.seed), w.prompt_len)
    print(f"{name}: batched prefill of {w.prompt_len} positions {ms:.1f} ms")

"""Edge cases of the decode path through the C ABI: short and long prompts,
several GQA shapes, chunk sizes, session control (continuation, rewind,
EOS, capacity), argument errors and the bounded-wait failure path."""
import numpy as np
import pytest

import synth
from oracle import OracleModel
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


def _session(shape, dev, max_seq, eos=-1):
    from persistent_sm_decode_monokernel_b200 import Session
    return Session(shape, dev, max_seq=max_seq, eos_id=eos)


def _forced_parity(shape, prompt_len, n, seed=0, options=()):
    m = synth.make_model(shape, seed=seed)
    prompt = synth.make_prompt(shape.vocab, prompt_len, seed=seed)
    forced = synth.make_forced_ids(shape.vocab, n, seed=seed)
    s = _session(shape, device_model(m), prompt_len + n)
    for opt, val in options:
        s.set_option(opt, val)
    cap0 = s.capture_logits(1)
    g0 = s.prefill(prompt)
    l0 = cap0.cpu().numpy().copy()
    cap = s.capture_logits(n)
    picks = s.decode_forced(forced)
    lg = np.concatenate([l0, cap.cpu().numpy()])
    s.close()
    seq = np.concatenate([prompt, forced])
    ref = OracleModel(m, dtype=np.float32).forward(seq, logits_rows=range(prompt_len - 1, len(seq)))
    return compare_steps(lg, np.concatenate([[g0], picks]), ref)


SHAPES = {
    # GQA group 8, head_dim 64, d 512 (2 pieces), ffn 1280 (5 pieces)
    "g8-hd64": synth.ModelShape(2, 512, 16, 2, 64, 1280, 3001),
    # GQA group 2, head_dim 128, d 768 (3 pieces), odd vocab
    "g2-hd128": synth.ModelShape(3, 768, 6, 3, 128, 2048, 4097),
    # group 5 like the 2.2B model, 2 layers
    "g5-hd128": synth.ModelShape(2, 1280, 10, 2, 128, 3584, 5000, rope_base=500000.0),
    # multi-query (one KV head), group 4
    "mqa-hd64": synth.ModelShape(2, 256, 4, 1, 64, 768, 1000),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_gqa_shapes_forced_parity(torch_cuda, name):
    rep = _forced_parity(SHAPES[name], 37, 24)
    assert rep.id_checked > 0


def test_single_token_prompt(torch_cuda):
    rep = _forced_parity(synth.WORKLOADS["tiny-l2-d256"].shape, 1, 12)
    assert rep.compared == 13


def test_long_context_many_splits(torch_cuda):
    # 1000-position prompt: 16 attention splits per KV head
    rep = _forced_parity(synth.WORKLOADS["tiny-l2-d256"].shape, 1000, 16)
    assert rep.compared == 17


def test_long_context_one_split_many_blocks(torch_cuda):
    # one split over ~1000 positions: online softmax across 256-position blocks
    from persistent_sm_decode_monokernel_b200 import _kie
    rep = _forced_parity(synth.WORKLOADS["tiny-l2-d256"].shape, 1000, 8,
                         options=[(_kie.KIE_OPT_MIN_SPLIT_LEN, 4096)])
    assert rep.compared == 9


@pytest.mark.parametrize("chunk", [8192, 12800, 65536, 98304])
def test_chunk_sizes(torch_cuda, chunk):
    from persistent_sm_decode_monokernel_b200 import _kie
    rep = _forced_parity(synth.WORKLOADS["l16-d1024"].shape, 40, 12,
                         options=[(_kie.KIE_OPT_CHUNK_BYTES, chunk)])
    assert rep.compared == 13


@pytest.fixture(scope="module")
def tiny(torch_cuda):
    w = synth.WORKLOADS["tiny-l2-d256"]
    m = synth.make_model(w.shape, seed=0)
    return w, m, device_model(m), synth.make_prompt(w.shape.vocab, w.prompt_len, seed=0)


def test_decode_continues_across_calls_and_rewind_repeats(tiny):
    w, m, dev, prompt = tiny
    s = _session(w.shape, dev, 64)
    s.prefill(prompt)
    a = list(s.decode(10))
    s.rewind(len(prompt))
    b = list(s.decode(4)) + list(s.decode(6))
    s.rewind(len(prompt))
    c = list(s.decode(10))
    assert a == b == c
    assert s.stats()["pos"] == len(prompt) + 10
    s.close()


def test_zero_steps_and_state_errors(tiny):
    from persistent_sm_decode_monokernel_b200 import KieError, _kie
    w, m, dev, prompt = tiny
    s = _session(w.shape, dev, 20)
    with pytest.raises(KieError) as e:
        s.decode(3)
    assert e.value.status == _kie.KIE_ERR_STATE
    s.prefill(prompt)
    assert len(s.decode(0)) == 0
    with pytest.raises(KieError) as e:
        s.decode(5)                       # 16 + 5 > 20 positions
    assert e.value.status == _kie.KIE_ERR_CAPACITY
    assert len(s.decode(4)) == 4          # capacity errors leave the context usable
    with pytest.raises(KieError) as e:
        s.prefill([w.shape.vocab])        # id out of range
    assert e.value.status == _kie.KIE_ERR_INVALID_ARG
    with pytest.raises(KieError) as e:
        s.rewind(0)
    assert e.value.status == _kie.KIE_ERR_INVALID_ARG
    s.close()


def test_eos_stops_decode(tiny):
    w, m, dev, prompt = tiny
    s = _session(w.shape, dev, 64)
    s.prefill(prompt)
    ids = list(s.decode(20))
    s.close()
    k = 6
    eos = ids[k]
    first = ids.index(eos)
    s2 = _session(w.shape, dev, 64, eos=eos)
    s2.prefill(prompt)
    out = list(s2.decode(20))
    assert out == ids[:first + 1]
    assert s2.stats()["pos"] == len(prompt) + first + 1
    s2.close()


def test_withheld_publication_times_out_and_context_fails(tiny, torch_cuda):
    from persistent_sm_decode_monokernel_b200 import KieError, _kie
    w, m, dev, prompt = tiny
    s = _session(w.shape, dev, 64)
    s.prefill(prompt)
    s.set_option(_kie.KIE_OPT_TIMEOUT_NS, 50_000_000)   # 50 ms per wait
    s.set_option(_kie.KIE_OPT_FAULT_CTA, 3)
    s.set_option(_kie.KIE_OPT_FAULT_STEP, 1)
    s.set_option(_kie.KIE_OPT_FAULT_LAYER, 1)
    s.set_option(_kie.KIE_OPT_FAULT_STAGE, _kie.STAGE_GU)
    with pytest.raises(KieError) as e:
        s.decode(4)
    assert e.value.status == _kie.KIE_ERR_TIMEOUT
    with pytest.raises(KieError) as e:
        s.decode(1)
    assert e.value.status == _kie.KIE_ERR_STATE
    s.close()
    torch_cuda.cuda.synchronize()
    # the device is healthy: a fresh context decodes normally
    s2 = _session(w.shape, dev, 64)
    s2.prefill(prompt)
    assert len(s2.decode(4)) == 4
    s2.close()


def test_stats_after_decode(tiny):
    w, m, dev, prompt = tiny
    s = _session(w.shape, dev, 64)
    s.prefill(prompt)
    s.decode(8)
    st = s.stats()
    assert st["grid"] >= 1 and st["ring_bytes"] >= 2 * st["chunk_bytes"]
    assert st["last_steps"] == 8 and st["last_device_ms"] > 0
    assert 0 <= st["sync_wait_cycles"] <= st["loop_cycles"]
    s.close()


def test_l2_prefetch_option_keeps_parity(torch_cuda):
    from persistent_sm_decode_monokernel_b200 import _kie
    rep = _forced_parity(synth.WORKLOADS["l16-d1024"].shape, 40, 12,
                         options=[(_kie.KIE_OPT_L2_PREFETCH_BYTES, 131072)])
    assert rep.compared == 13


@pytest.mark.parametrize("park", [0, 1])
def test_tmem_park_option_keeps_parity(torch_cuda, park):
    # on (the default): the chunks a warp parked while it waited are read
    # back from tensor memory; off: every chunk is read from the ring
    from persistent_sm_decode_monokernel_b200 import _kie
    rep = _forced_parity(synth.WORKLOADS["l16-d1024"].shape, 300, 12,
                         options=[(_kie.KIE_OPT_TMEM_PARK, park)])
    assert rep.compared == 13


def test_trace_of_every_cta(tiny):
    from persistent_sm_decode_monokernel_b200 import TRACE_PER_LAYER
    w, m, dev, prompt = tiny
    s = _session(w.shape, dev, 64)
    s.prefill(prompt)
    grid = s.stats()["grid"]
    buf = s.trace(3, -1)
    assert tuple(buf.shape) == (3, grid, w.shape.n_layers * TRACE_PER_LAYER + 4)
    s.decode(3)
    t = buf.cpu().numpy().astype(np.int64)
    s.trace_off()
    s.close()
    L = w.shape.n_layers
    for step in range(3):
        for c in range(grid):
            row = t[step, c]
            for l in range(L):
                e = row[l * TRACE_PER_LAYER:]
                # QKV begin <= QKV done <= attention done <= O done <= gate/up done <= down done
                stamps = [e[0], e[2], e[3], e[5], e[7], e[9]]
                assert all(x > 0 for x in stamps), (step, c, l)
                assert stamps == sorted(stamps), (step, c, l, stamps)
            lm = row[L * TRACE_PER_LAYER:L * TRACE_PER_LAYER + 4]
            assert lm[0] > 0 and lm[3] >= lm[0]

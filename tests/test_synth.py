"""The seeded input generator: deterministic, shaped and distributed as stated."""
import numpy as np

import synth


def _shape():
    return synth.ModelShape(2, 64, 4, 2, 16, 96, 97)


def test_deterministic_and_thread_independent():
    a = synth.make_model(_shape(), seed=1, threads=1)
    b = synth.make_model(_shape(), seed=1, threads=8)
    assert list(a.tensors) == synth.tensor_names(2)
    for k in a.tensors:
        assert a[k].dtype == np.float16
        np.testing.assert_array_equal(a[k], b[k])


def test_seed_changes_weights():
    a = synth.make_model(_shape(), seed=1)
    b = synth.make_model(_shape(), seed=2)
    assert not np.array_equal(a["0.wq"], b["0.wq"])


def test_shapes_gains_and_distribution():
    s = synth.WORKLOADS["tiny-l2-d256"].shape
    m = synth.make_model(s, seed=0)
    assert m["tok_emb"].shape == (2048, 256)
    assert m["0.wq"].shape == (256, 256) and m["0.wk"].shape == (256, 256)
    assert m["0.wo"].shape == (256, 256)
    assert m["1.w_down"].shape == (256, 768) and m["1.w_up"].shape == (768, 256)
    for n in ("0.attn_norm", "0.ffn_norm", "final_norm"):
        assert np.all(m[n] == 1.0)
    x = m["lm_head"].astype(np.float64)
    assert abs(x.mean()) < 2e-4
    assert abs(x.std() - 0.02) < 2e-4


def test_prompt_and_forced_ids():
    p = synth.make_prompt(2048, 16, seed=0)
    assert p.dtype == np.int32 and p.shape == (16,)
    assert p.min() >= 0 and p.max() < 2048
    np.testing.assert_array_equal(p, synth.make_prompt(2048, 16, seed=0))
    f = synth.make_forced_ids(2048, 16, seed=0)
    assert not np.array_equal(p, f)


def test_workload_byte_counts():
    w = synth.WORKLOADS["l28-d2560"]
    assert abs(w.shape.n_params() - 2.184e9) / 2.184e9 < 2e-3
    assert w.shape.kv_bytes_per_position() == 57344
    # ~4.11 GB of weights + ~58.8 MB of KV per token at the mean position
    assert abs(w.bytes_per_token_mean() / 1e6 - 4170.2) < 3.0

"""Pins of the CPU oracle to things other than itself.

Each test checks one oracle function against a closed form, an invariant,
a special case that reduces to a textbook result, or brute force on tiny
inputs, chosen so that a plausible slip (a dropped residual, a swapped gate
and up, a wrong softmax scale, the wrong RoPE pairing or sign, an off-by-one
causal mask, interleaved GQA groups, a missing norm gain) fails at least one.
The worked inputs live in tests/golden/closed_forms.json.
"""
import json
import math
import os

import numpy as np
import pytest

import synth
from oracle import (OracleModel, apply_rope, argmax_lowest, attention_one_query,
                    causal_attention, rms_norm, rope_cos_sin, rope_inv_freq,
                    silu, top2_margin)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _tiny_shape(**kw):
    base = dict(n_layers=2, d_model=64, n_heads=4, n_kv_heads=2, head_dim=16,
                ffn_dim=96, vocab=97)
    base.update(kw)
    return synth.ModelShape(**base)


def _random_gains(model, seed=5):
    rng = np.random.default_rng(seed)
    for k in list(model.tensors):
        if k.endswith("norm"):
            n = model.tensors[k].shape[0]
            model.tensors[k] = (1.0 + 0.5 * rng.standard_normal(n)).astype(np.float16)
    return model


# ------------------------------------------------------------------ RMSNorm

def test_rmsnorm_unit_gain_closed_form():
    rng = np.random.default_rng(0)
    for eps in (1e-5, 0.3):
        x = rng.standard_normal((7, 33)) * rng.uniform(0.01, 5, size=(7, 1))
        y = rms_norm(x, np.ones(33), eps)
        ms = np.mean(x * x, axis=1)
        got = np.sqrt(np.mean(y * y, axis=1))
        np.testing.assert_allclose(got, np.sqrt(ms / (ms + eps)), rtol=1e-13)


def test_rmsnorm_hand_example():
    g = _golden()["rmsnorm"]
    x = np.array(g["x"], dtype=np.float64)
    y = rms_norm(x, np.array(g["gain"], dtype=np.float64), g["eps"])
    # mean(x^2) = (9 + 16) / 2 = 12.5; sqrt(12.5 + 0.5) = sqrt(13)
    want = [2.0 * 3.0 / math.sqrt(13.0), 0.5 * 4.0 / math.sqrt(13.0)]
    np.testing.assert_allclose(y, want, rtol=1e-15)


def test_rmsnorm_scale_invariant_without_eps():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(50)
    gain = rng.standard_normal(50)
    np.testing.assert_allclose(rms_norm(37.5 * x, gain, 0.0), rms_norm(x, gain, 0.0),
                               rtol=1e-13)


def test_rmsnorm_float32_stays_float32():
    x = np.ones(8, dtype=np.float32)
    assert rms_norm(x, np.ones(8, dtype=np.float32), 1e-5).dtype == np.float32


# --------------------------------------------------------------------- RoPE

def test_rope_inv_freq_closed_form():
    th = rope_inv_freq(128, 10000.0)
    assert th[0] == 1.0
    assert math.isclose(th[1], 10000.0 ** (-2.0 / 128), rel_tol=1e-15)
    assert math.isclose(th[63], 10000.0 ** (-126.0 / 128), rel_tol=1e-14)


def test_rope_identity_at_position_zero():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 64))
    c, s = rope_cos_sin([0], 64, 10000.0)
    np.testing.assert_array_equal(apply_rope(x, c, s), x)


def test_rope_hand_example_half_split_pairs():
    g = _golden()["rope"]
    c, s = rope_cos_sin([g["pos"]], g["head_dim"], g["base"])
    y = apply_rope(np.array(g["x"], dtype=np.float64), c[0], s[0])
    # theta = [1, 100^-0.5 = 0.1]; angles [2, 0.2]; pairs (0,2) and (1,3)
    a0, a1 = 2.0, 0.2
    want = [1 * math.cos(a0) - 3 * math.sin(a0),
            2 * math.cos(a1) - 4 * math.sin(a1),
            3 * math.cos(a0) + 1 * math.sin(a0),
            4 * math.cos(a1) + 2 * math.sin(a1)]
    np.testing.assert_allclose(y, want, rtol=1e-14, atol=1e-15)


def test_rope_head_dim_two_is_plane_rotation():
    for t in (1, 5, 1000):
        c, s = rope_cos_sin([t], 2, 10000.0)
        x = np.array([0.3, -1.7])
        R = np.array([[math.cos(t), -math.sin(t)], [math.sin(t), math.cos(t)]])
        np.testing.assert_allclose(apply_rope(x, c[0], s[0]), R @ x, rtol=1e-12, atol=1e-14)


def test_rope_preserves_pair_norms():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(128)
    c, s = rope_cos_sin([777], 128, 500000.0)
    y = apply_rope(x, c[0], s[0])
    n_in = x[:64] ** 2 + x[64:] ** 2
    n_out = y[:64] ** 2 + y[64:] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12)


def test_rope_relative_position_invariance():
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in ((9, 2), (300, 300), (4096, 17)):
        cm, sm = rope_cos_sin([m], 64, 10000.0)
        cn, sn = rope_cos_sin([n], 64, 10000.0)
        cd, sd = rope_cos_sin([m - n], 64, 10000.0)
        lhs = apply_rope(q, cm[0], sm[0]) @ apply_rope(k, cn[0], sn[0])
        rhs = apply_rope(q, cd[0], sd[0]) @ k
        assert math.isclose(lhs, rhs, rel_tol=1e-9, abs_tol=1e-9)


# -------------------------------------------------------------------- SiLU

def test_silu_values():
    z = np.array([0.0, 1.0, -1.0, 30.0, -30.0])
    y = silu(z)
    assert y[0] == 0.0
    assert math.isclose(y[1], 1.0 / (1.0 + math.exp(-1.0)), rel_tol=1e-15)
    assert math.isclose(y[2], -1.0 / (1.0 + math.exp(1.0)), rel_tol=1e-15)
    assert math.isclose(y[3], 30.0, rel_tol=1e-12)
    assert abs(y[4]) < 1e-11


# ---------------------------------------------------------------- attention

def test_attention_single_position_returns_its_value():
    rng = np.random.default_rng(5)
    q, K, V = rng.standard_normal(16), rng.standard_normal((1, 16)), rng.standard_normal((1, 16))
    np.testing.assert_allclose(attention_one_query(q, K, V), V[0], rtol=1e-15)


def test_attention_identical_keys_average_values():
    rng = np.random.default_rng(6)
    q = rng.standard_normal(16)
    K = np.tile(rng.standard_normal(16), (9, 1))
    V = rng.standard_normal((9, 16))
    np.testing.assert_allclose(attention_one_query(q, K, V), V.mean(axis=0), rtol=1e-12, atol=1e-14)


def test_attention_two_positions_closed_form_scale():
    g = _golden()["attention_two_positions"]
    q = np.array(g["q"], dtype=np.float64)
    K = np.array(g["K"], dtype=np.float64)
    V = np.array(g["V"], dtype=np.float64)
    # scores: q.k0 / sqrt(4) = 2/2 = 1, q.k1 / 2 = 0  ->  p0 = e / (e + 1)
    p0 = math.e / (math.e + 1.0)
    want = p0 * V[0] + (1.0 - p0) * V[1]
    np.testing.assert_allclose(attention_one_query(q, K, V), want, rtol=1e-14)


def _attention_bruteforce(q, k, v):
    T, H, hd = q.shape
    KV = k.shape[1]
    G = H // KV
    out = np.zeros_like(q)
    for t in range(T):
        for h in range(H):
            j = h // G
            s = [sum(q[t, h, e] * k[u, j, e] for e in range(hd)) / math.sqrt(hd)
                 for u in range(t + 1)]
            mx = max(s)
            w = [math.exp(x - mx) for x in s]
            z = sum(w)
            for e in range(hd):
                out[t, h, e] = sum(w[u] * v[u, j, e] for u in range(t + 1)) / z
    return out


def test_causal_attention_matches_bruteforce_loops():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((5, 4, 4))
    k = rng.standard_normal((5, 2, 4))
    v = rng.standard_normal((5, 2, 4))
    np.testing.assert_allclose(causal_attention(q, k, v), _attention_bruteforce(q, k, v),
                               rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------ whole model

def test_incremental_equals_full_sequence_fp64():
    m = _random_gains(synth.make_model(_tiny_shape(), seed=3))
    om = OracleModel(m, dtype=np.float64)
    toks = synth.make_prompt(97, 12, seed=3)
    full = om.forward(toks)
    st = om.new_state()
    inc = np.stack([om.decode_step(st, t) for t in toks])
    np.testing.assert_allclose(inc, full, rtol=1e-11, atol=1e-12)


def test_batched_prefill_state_equals_incremental():
    m = synth.make_model(_tiny_shape(), seed=4)
    om = OracleModel(m, dtype=np.float64)
    prompt = synth.make_prompt(97, 9, seed=4)
    st_a = om.new_state()
    lg_a = om.prefill(st_a, prompt)
    st_b, lg_b = om.prefill_batched(prompt)
    np.testing.assert_allclose(lg_b, lg_a, rtol=1e-11, atol=1e-12)
    nxt = argmax_lowest(lg_a)
    np.testing.assert_allclose(om.decode_step(st_b, nxt), om.decode_step(st_a, nxt),
                               rtol=1e-11, atol=1e-12)


def test_causality_future_tokens_do_not_change_past_logits():
    m = synth.make_model(_tiny_shape(), seed=5)
    om = OracleModel(m, dtype=np.float64)
    a = synth.make_prompt(97, 10, seed=5)
    b = a.copy()
    b[6:] = (b[6:] + 11) % 97
    la, lb = om.forward(a), om.forward(b)
    np.testing.assert_allclose(la[:6], lb[:6], rtol=1e-13, atol=1e-14)
    assert np.max(np.abs(la[6:] - lb[6:])) > 1e-3


def test_gqa_equals_mha_with_kv_heads_repeated_per_group():
    shp = _tiny_shape(n_heads=4, n_kv_heads=2)
    m = synth.make_model(shp, seed=6)
    G, hd = 2, shp.head_dim
    mha_shape = _tiny_shape(n_heads=4, n_kv_heads=4)
    over = {}
    for l in range(shp.n_layers):
        for w in ("wk", "wv"):
            src = m[f"{l}.{w}"].reshape(2, hd, shp.d_model)
            over[f"{l}.{w}"] = np.repeat(src, G, axis=0).reshape(4 * hd, shp.d_model)
    mha = synth.SynthModel(mha_shape, 6, dict(m.tensors))
    mha.tensors.update(over)
    toks = synth.make_prompt(97, 8, seed=6)
    la = OracleModel(m, dtype=np.float64).forward(toks)
    lb = OracleModel(mha, dtype=np.float64).forward(toks)
    np.testing.assert_allclose(la, lb, rtol=1e-12, atol=1e-13)


def _norm64(x, g, eps):
    return g * x / math.sqrt(float(np.mean(x * x)) + eps)


def test_zero_blocks_reduce_to_embedding_lm_head():
    shp = _tiny_shape()
    m = _random_gains(synth.make_model(shp, seed=7))
    for l in range(shp.n_layers):
        m.tensors[f"{l}.wo"][:] = 0
        m.tensors[f"{l}.w_down"][:] = 0
    om = OracleModel(m, dtype=np.float64)
    toks = [5, 60, 5, 96]
    got = om.forward(toks)
    E = m["tok_emb"].astype(np.float64)
    W = m["lm_head"].astype(np.float64)
    gf = m["final_norm"].astype(np.float64)
    want = np.stack([W @ _norm64(E[t], gf, shp.rms_eps) for t in toks])
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def test_attention_branch_single_position_closed_form():
    # one token, one layer, FFN output zeroed: attention over one position
    # returns v, so h = E + Wo concat_h(v_{j(h)}), v = Wv RMSNorm(E; g_attn).
    shp = _tiny_shape(n_layers=1, n_heads=4, n_kv_heads=2)
    m = _random_gains(synth.make_model(shp, seed=8))
    m.tensors["0.w_down"][:] = 0
    om = OracleModel(m, dtype=np.float64)
    tok = 42
    E = m["tok_emb"].astype(np.float64)[tok]
    a = _norm64(E, m["0.attn_norm"].astype(np.float64), shp.rms_eps)
    v = (m["0.wv"].astype(np.float64) @ a).reshape(2, shp.head_dim)
    o = np.concatenate([v[0], v[0], v[1], v[1]])
    h = E + m["0.wo"].astype(np.float64) @ o
    want = m["lm_head"].astype(np.float64) @ _norm64(h, m["final_norm"].astype(np.float64),
                                                     shp.rms_eps)
    np.testing.assert_allclose(om.forward([tok])[0], want, rtol=1e-12, atol=1e-13)


def test_ffn_branch_closed_form_gate_gets_silu():
    shp = _tiny_shape(n_layers=1)
    m = _random_gains(synth.make_model(shp, seed=9))
    m.tensors["0.wo"][:] = 0
    om = OracleModel(m, dtype=np.float64)
    tok = 13
    E = m["tok_emb"].astype(np.float64)[tok]
    b = _norm64(E, m["0.ffn_norm"].astype(np.float64), shp.rms_eps)
    gz = m["0.w_gate"].astype(np.float64) @ b
    uz = m["0.w_up"].astype(np.float64) @ b
    act = np.array([z / (1.0 + math.exp(-z)) for z in gz]) * uz
    h = E + m["0.w_down"].astype(np.float64) @ act
    want = m["lm_head"].astype(np.float64) @ _norm64(h, m["final_norm"].astype(np.float64),
                                                     shp.rms_eps)
    np.testing.assert_allclose(om.forward([tok])[0], want, rtol=1e-12, atol=1e-13)


def _one_layer_scalar_loops(m, toks):
    """Logits of a one-layer model at every position of `toks`, written as
    scalar loops straight from the block's definition (no numpy algebra):
    q_h from rows h*hd .. h*hd+hd-1 of Wq, k_j and v_j likewise from Wk and
    Wv, RoPE on q AND k at the token's own position t (pairs (i, i+hd/2),
    angle t * base^(-2i/hd)), scores over u <= t scaled by 1/sqrt(hd),
    softmax, weighted sum of v, Wo, residual, RMSNorm, SwiGLU FFN, residual,
    final RMSNorm and the LM head.  Python floats are IEEE doubles."""
    s = m.shape
    d, H, KV, hd, F, V = s.d_model, s.n_heads, s.n_kv_heads, s.head_dim, s.ffn_dim, s.vocab
    G, half, eps = H // KV, hd // 2, s.rms_eps
    f = {k: v.astype(np.float64).tolist() for k, v in m.tensors.items()}

    def norm(x, g):
        ms = sum(xi * xi for xi in x) / len(x)
        r = 1.0 / math.sqrt(ms + eps)
        return [g[c] * x[c] * r for c in range(len(x))]

    def matvec(W, x):
        return [sum(W[r][c] * x[c] for c in range(len(x))) for r in range(len(W))]

    def rope(vec, t):
        out = list(vec)
        for i in range(half):
            ang = t * s.rope_base ** (-2.0 * i / hd)
            c, sn = math.cos(ang), math.sin(ang)
            out[i] = vec[i] * c - vec[i + half] * sn
            out[i + half] = vec[i + half] * c + vec[i] * sn
        return out

    keys, vals, logits = [], [], []
    for t, tok in enumerate(toks):
        h = list(f["tok_emb"][tok])
        a = norm(h, f["0.attn_norm"])
        q = [rope([sum(f["0.wq"][hh * hd + i][c] * a[c] for c in range(d)) for i in range(hd)], t)
             for hh in range(H)]
        keys.append([rope([sum(f["0.wk"][j * hd + i][c] * a[c] for c in range(d))
                           for i in range(hd)], t) for j in range(KV)])
        vals.append([[sum(f["0.wv"][j * hd + i][c] * a[c] for c in range(d)) for i in range(hd)]
                     for j in range(KV)])
        o = []
        for hh in range(H):
            j = hh // G
            sc = [sum(q[hh][i] * keys[u][j][i] for i in range(hd)) / math.sqrt(hd)
                  for u in range(t + 1)]
            mx = max(sc)
            e = [math.exp(x - mx) for x in sc]
            z = sum(e)
            o += [sum(e[u] / z * vals[u][j][i] for u in range(t + 1)) for i in range(hd)]
        att = matvec(f["0.wo"], o)
        h = [h[r] + att[r] for r in range(d)]
        b = norm(h, f["0.ffn_norm"])
        gz, uz = matvec(f["0.w_gate"], b), matvec(f["0.w_up"], b)
        act = [gz[k] / (1.0 + math.exp(-gz[k])) * uz[k] for k in range(F)]
        dn = matvec(f["0.w_down"], act)
        h = [h[r] + dn[r] for r in range(d)]
        logits.append(matvec(f["lm_head"], norm(h, f["final_norm"])))
    return np.array(logits)


def _qk_pin_model():
    # weights ~N(0, 0.5) so that the softmax is far from uniform and the
    # rotation angles (1 and 2 rad at i = 0) move the scores
    shp = _tiny_shape(n_layers=1, d_model=16, n_heads=4, n_kv_heads=2, head_dim=8,
                      ffn_dim=12, vocab=11, rope_base=100.0)
    m = _random_gains(synth.make_model(shp, seed=12), seed=13)
    rng = np.random.default_rng(14)
    for k, v in m.tensors.items():
        if not k.endswith("norm"):
            m.tensors[k] = (0.5 * rng.standard_normal(v.shape)).astype(np.float16)
    return m


def test_one_layer_model_equals_scalar_loops_at_three_positions():
    # pins how rows of Wq / Wk / Wv map to heads, RoPE of both q and k at
    # each token's position, the causal range and GQA wiring at the model
    # level, in both oracle paths
    m = _qk_pin_model()
    toks = [3, 7, 3]
    want = _one_layer_scalar_loops(m, toks)
    om = OracleModel(m, dtype=np.float64)
    np.testing.assert_allclose(om.forward(toks), want, rtol=1e-12, atol=1e-12)
    st = om.new_state()
    inc = np.stack([om.decode_step(st, t) for t in toks])
    np.testing.assert_allclose(inc, want, rtol=1e-12, atol=1e-12)
    # the positions differ: a model that ignored q, k or the rotation would
    # give position 2 the logits of a one-token context of the same token
    assert np.max(np.abs(want[2] - want[0])) > 1e-2


def test_argmax_lowest_index_on_ties_bruteforce():
    rng = np.random.default_rng(10)
    for trial in range(50):
        x = rng.integers(-3, 4, size=40).astype(np.float32)
        best, bi = -np.inf, -1
        for i, v in enumerate(x):
            if v > best:
                best, bi = v, i
        assert argmax_lowest(x) == bi


def test_top2_margin():
    assert top2_margin(np.array([0.1, 3.0, 2.5, -1.0])) == pytest.approx(0.5)
    assert top2_margin(np.array([1.0, 1.0])) == 0.0


def test_greedy_is_self_consistent_and_stops_on_eos():
    m = synth.make_model(_tiny_shape(), seed=11)
    om = OracleModel(m, dtype=np.float64)
    prompt = synth.make_prompt(97, 6, seed=11)
    ids, lg = om.greedy(prompt, 10)
    assert len(ids) == 11 and lg.shape == (11, 97)
    assert ids == [int(np.argmax(r)) for r in lg]
    full = om.forward(list(prompt) + ids[:-1])
    np.testing.assert_allclose(full[len(prompt) - 1:], lg, rtol=1e-11, atol=1e-12)
    k = 4
    ids_e, _ = om.greedy(prompt, 10, eos_id=ids[k])
    first = ids.index(ids[k])
    assert ids_e == ids[:first + 1]


def test_float32_drift_against_float64_is_small():
    w = synth.WORKLOADS["tiny-l2-d256"]
    m = synth.make_model(w.shape, seed=0)
    toks = list(synth.make_prompt(w.shape.vocab, 24, seed=0))
    l32 = OracleModel(m, dtype=np.float32).forward(toks)
    l64 = OracleModel(m, dtype=np.float64).forward(toks)
    assert l32.dtype == np.float32
    err = np.max(np.abs(l32 - l64)) / np.max(np.abs(l64))
    assert err < 1e-5, err


def test_fp16_kv_rounding_changes_little():
    w = synth.WORKLOADS["tiny-l2-d256"]
    m = synth.make_model(w.shape, seed=0)
    toks = list(synth.make_prompt(w.shape.vocab, 24, seed=0))
    a = OracleModel(m, dtype=np.float64).forward(toks)
    b = OracleModel(m, dtype=np.float64, kv_fp16=True).forward(toks)
    rel = np.max(np.abs(a - b)) / np.max(np.abs(a))
    assert 0 < rel < 2e-3, rel

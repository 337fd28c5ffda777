"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin
catches each one.  This guards the pins themselves: a pin set that still
passes with a wrong RoPE pairing or a wrong softmax scale pins nothing.
"""
import math

import numpy as np
import pytest

import oracle.model as om
import test_oracle_pins as pins


def _rope_interleaved(x, cos, sin):
    c = cos.astype(x.dtype)
    s = sin.astype(x.dtype)
    x1, x2 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


def _rope_wrong_sign(x, cos, sin):
    return om.__dict__["_orig_apply_rope"](x, cos, -sin)


def _attn_one_scale_hd(q, K, V):
    s = (K @ q) / q.dtype.type(q.shape[-1])
    p = np.exp(s - np.max(s))
    return (p / p.sum()) @ V


def _causal_excludes_self(q, k, v):
    T, H, hd = q.shape
    G = H // k.shape[1]
    out = np.zeros_like(q)
    for h in range(H):
        j = h // G
        s = (q[:, h] @ k[:, j].T) / math.sqrt(hd)
        s[np.triu(np.ones((T, T), bool), k=0)] = -np.inf
        s[0, 0] = 0.0
        p = np.exp(s - s.max(1, keepdims=True))
        out[:, h] = (p / p.sum(1, keepdims=True)) @ v[:, j]
    return out


def _causal_interleaved_groups(q, k, v):
    T, H, hd = q.shape
    KV = k.shape[1]
    out = np.empty_like(q)
    mask = np.triu(np.ones((T, T), bool), k=1)
    for h in range(H):
        j = h % KV
        s = (q[:, h] @ k[:, j].T) / math.sqrt(hd)
        s[mask] = -np.inf
        p = np.exp(s - s.max(1, keepdims=True))
        out[:, h] = (p / p.sum(1, keepdims=True)) @ v[:, j]
    return out


def _rms_no_gain(x, gain, eps):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def _rms_no_eps(x, gain, eps):
    return gain * x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True))


def _silu_sigmoid_only(z):
    return 1.0 / (1.0 + np.exp(-z))


MUTATIONS = [
    ("apply_rope", _rope_interleaved, pins.test_rope_hand_example_half_split_pairs),
    ("apply_rope", _rope_wrong_sign, pins.test_rope_hand_example_half_split_pairs),
    ("attention_one_query", _attn_one_scale_hd, pins.test_attention_two_positions_closed_form_scale),
    ("causal_attention", _causal_excludes_self, pins.test_causal_attention_matches_bruteforce_loops),
    ("causal_attention", _causal_interleaved_groups, pins.test_gqa_equals_mha_with_kv_heads_repeated_per_group),
    ("rms_norm", _rms_no_gain, pins.test_zero_blocks_reduce_to_embedding_lm_head),
    ("rms_norm", _rms_no_eps, pins.test_rmsnorm_unit_gain_closed_form),
    ("silu", _silu_sigmoid_only, pins.test_silu_values),
    ("silu", _silu_sigmoid_only, pins.test_ffn_branch_closed_form_gate_gets_silu),
]


@pytest.mark.parametrize("name,bad,pin", MUTATIONS,
                         ids=[f"{m[0]}:{m[1].__name__}->{m[2].__name__}" for m in MUTATIONS])
def test_pin_catches_planted_mistake(monkeypatch, name, bad, pin):
    monkeypatch.setitem(om.__dict__, "_orig_apply_rope", om.apply_rope)
    monkeypatch.setattr(om, name, bad)
    monkeypatch.setattr(pins, name, bad, raising=False)
    with pytest.raises(AssertionError):
        pin()


# ---- mistakes in the model-level wiring of q and k (both oracle paths)

def _k_cached_without_rope():
    # both paths call apply_rope for q, then for k, in every layer and step:
    # rotate the odd calls only, so k enters the cache unrotated
    orig = om.apply_rope
    calls = [0]

    def rope(x, cos, sin):
        calls[0] += 1
        return orig(x, cos, sin) if calls[0] % 2 == 1 else x
    return rope


def _q_reshaped_hd_by_h():
    # q = (Wq a).reshape(hd, H).T: head h dim i read from element i*H + h,
    # the same as Wq's rows permuted that way in both paths
    orig = om.OracleModel.w

    def w(self, name):
        a = orig(self, name)
        if name.endswith(".wq"):
            perm = [i * self.H + h for h in range(self.H) for i in range(self.hd)]
            a = a[perm]
        return a
    return w


MODEL_MUTATIONS = [
    ("apply_rope", _k_cached_without_rope),
    ("OracleModel.w", _q_reshaped_hd_by_h),
]


@pytest.mark.parametrize("name,make", MODEL_MUTATIONS, ids=[m[1].__name__ for m in MODEL_MUTATIONS])
def test_scalar_loop_pin_catches_model_level_mistake(monkeypatch, name, make):
    bad = make()
    if name == "OracleModel.w":
        monkeypatch.setattr(om.OracleModel, "w", bad)
    else:
        monkeypatch.setattr(om, name, bad)
    with pytest.raises(AssertionError):
        pins.test_one_layer_model_equals_scalar_loops_at_three_positions()

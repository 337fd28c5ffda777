"""CPU oracle for batch-1 greedy decode of a dense decoder-only transformer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only the tests, the smoke check and the benchmark's CPU-baseline leg do.
It shares no code with the CUDA path; both are fed the same seeded host
buffers from the `synth` module.

What it computes.  The pages describe one resident GPU program that runs the
whole decode loop -- prefill, decode, LM-head token selection and the EOS
check -- without returning to the CPU (revietech.ru, "Kog выжимает максимум из
GPU: 3000 токенов/с", section "Что такое monokernel"), whose projections are
matrix-vector products (same page, section "Архитектура и особенности",
"GEMV вместо GEMM").  The pages never print the model; the readings taken
here are the plain pre-norm (Llama-style) decoder block:

    h   = E[token]
    per layer:
        a   = RMSNorm(h; g_attn)
        q_h = Wq_h a,  k_j = Wk_j a,  v_j = Wv_j a          (head h, kv head j)
        q, k rotated by RoPE at the token's 0-based position (half-split pairs)
        o_h = sum_u softmax_u(q_h . k_{j(h),u} / sqrt(hd)) v_{j(h),u},  u <= t
        h  += Wo concat_h(o_h)
        b   = RMSNorm(h; g_ffn)
        h  += Wd (silu(Wg b) * (Wu b))
    logits = Wlm RMSNorm(h; g_final);   next = argmax(logits) (lowest index on ties)

with j(h) = floor(h / (H / KV)) (contiguous query-head groups per KV head),
RMSNorm(x; g) = g * x / sqrt(mean(x^2) + eps), silu(z) = z / (1 + e^-z),
RoPE angle t * base^(-2i/hd) applied to the pair (i, i + hd/2), i < hd/2,
computed in float64.  No biases, no embedding scale, untied LM head.

Precision: arithmetic in `dtype` (float32 by default, float64 for drift
bounds) on the exact fp16 weight values.  The KV cache holds `dtype` values;
`kv_fp16=True` rounds cached K and V to fp16 to mirror an fp16 cache.

Two independent code paths:
  * `forward`  -- whole sequence at once, causal mask, no cache;
  * `prefill` / `decode_step` -- one position at a time with a KV cache.
The tests pin them against each other and against closed forms.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "rms_norm", "rope_inv_freq", "rope_cos_sin", "apply_rope", "silu",
    "attention_one_query", "causal_attention", "argmax_lowest",
    "top2_margin", "OracleModel", "DecodeState",
]


# ---------------------------------------------------------------- primitives

def rms_norm(x: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """g * x / sqrt(mean(x^2) + eps) over the last axis."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return gain * (x / np.sqrt(ms + x.dtype.type(eps)))


def rope_inv_freq(head_dim: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/hd), i = 0 .. hd/2-1, in float64."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(base), -2.0 * i / head_dim)


def rope_cos_sin(positions: Sequence[int], head_dim: int, base: float):
    """cos and sin of t * theta_i for each position t, float64, [T, hd/2]."""
    t = np.asarray(positions, dtype=np.float64)
    ang = np.outer(t, rope_inv_freq(head_dim, base))
    return np.cos(ang), np.sin(ang)


def apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate the pairs (i, i + hd/2) of the last axis by the given angles.

    x: [..., hd]; cos, sin: broadcastable to [..., hd/2].
    out_i        = x_i cos - x_{i+hd/2} sin
    out_{i+hd/2} = x_{i+hd/2} cos + x_i sin
    """
    half = x.shape[-1] // 2
    c = cos.astype(x.dtype)
    s = sin.astype(x.dtype)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(z: np.ndarray) -> np.ndarray:
    one = z.dtype.type(1.0)
    return z / (one + np.exp(-z))


def attention_one_query(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """softmax(q K^T / sqrt(hd)) V for one query q [hd] over K, V [n, hd]."""
    hd = q.shape[-1]
    s = (K @ q) / q.dtype.type(math.sqrt(hd))
    s = s - np.max(s)
    p = np.exp(s)
    p = p / np.sum(p)
    return p @ V


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Full-sequence causal attention with grouped KV heads.

    q [T, H, hd], k and v [T, KV, hd]; query head h reads KV head h // (H/KV).
    Position t attends to positions 0..t.  Returns [T, H, hd].
    """
    T, H, hd = q.shape
    KV = k.shape[1]
    G = H // KV
    out = np.empty_like(q)
    scale = q.dtype.type(1.0 / math.sqrt(hd))
    future = np.triu(np.ones((T, T), dtype=bool), k=1)
    for h in range(H):
        j = h // G
        s = (q[:, h, :] @ k[:, j, :].T) * scale          # [T, T]
        s[future] = -np.inf
        s = s - np.max(s, axis=1, keepdims=True)
        p = np.exp(s)
        p = p / np.sum(p, axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, j, :]
    return out


def argmax_lowest(logits: np.ndarray) -> int:
    """Greedy pick: the largest logit, the lowest index among equal maxima."""
    return int(np.argmax(logits))


def top2_margin(logits: np.ndarray) -> float:
    """top-1 minus top-2 logit (absolute units)."""
    part = np.partition(np.asarray(logits, dtype=np.float64), -2)
    return float(part[-1] - part[-2])


# ---------------------------------------------------------------- the model

class DecodeState:
    """Per-layer KV cache of the incremental path: lists of [t, KV, hd]."""

    def __init__(self, n_layers: int):
        self.k: List[List[np.ndarray]] = [[] for _ in range(n_layers)]
        self.v: List[List[np.ndarray]] = [[] for _ in range(n_layers)]
        self.pos = 0


class OracleModel:
    """The transformer of the module docstring over a `synth.SynthModel`."""

    def __init__(self, model, dtype=np.float32, kv_fp16: bool = False,
                 cache_weights: bool = True):
        self.src = model
        s = model.shape
        self.shape = s
        self.dtype = np.dtype(dtype)
        self.kv_fp16 = kv_fp16
        self.L, self.d = s.n_layers, s.d_model
        self.H, self.KV, self.hd = s.n_heads, s.n_kv_heads, s.head_dim
        self.eps = s.rms_eps
        self._cache: Dict[str, np.ndarray] = {}
        self._cache_on = cache_weights

    # weights in the oracle's dtype
    def w(self, name: str) -> np.ndarray:
        a = self._cache.get(name)
        if a is None:
            a = self.src[name].astype(self.dtype)
            if self._cache_on:
                self._cache[name] = a
        return a

    def _kv_round(self, x: np.ndarray) -> np.ndarray:
        if self.kv_fp16:
            return x.astype(np.float16).astype(self.dtype)
        return x

    # ---- full-sequence path (no cache)
    def forward(self, tokens: Sequence[int],
                logits_rows: Optional[Sequence[int]] = None) -> np.ndarray:
        """Logits for every position of `tokens` (or only `logits_rows`)."""
        toks = np.asarray(tokens, dtype=np.int64)
        T = toks.shape[0]
        h = self.w("tok_emb")[toks]                                  # [T, d]
        cos, sin = rope_cos_sin(range(T), self.hd, self.shape.rope_base)
        cos, sin = cos[:, None, :], sin[:, None, :]
        for l in range(self.L):
            p = f"{l}."
            a = rms_norm(h, self.w(p + "attn_norm"), self.eps)
            q = (a @ self.w(p + "wq").T).reshape(T, self.H, self.hd)
            k = (a @ self.w(p + "wk").T).reshape(T, self.KV, self.hd)
            v = (a @ self.w(p + "wv").T).reshape(T, self.KV, self.hd)
            q = apply_rope(q, cos, sin)
            k = self._kv_round(apply_rope(k, cos, sin))
            v = self._kv_round(v)
            o = causal_attention(q, k, v).reshape(T, self.H * self.hd)
            h = h + o @ self.w(p + "wo").T
            b = rms_norm(h, self.w(p + "ffn_norm"), self.eps)
            g = b @ self.w(p + "w_gate").T
            u = b @ self.w(p + "w_up").T
            h = h + (silu(g) * u) @ self.w(p + "w_down").T
        if logits_rows is not None:
            h = h[np.asarray(logits_rows, dtype=np.int64)]
        hn = rms_norm(h, self.w("final_norm"), self.eps)
        return hn @ self.w("lm_head").T

    # ---- incremental path (KV cache, one position per call)
    def new_state(self) -> DecodeState:
        return DecodeState(self.L)

    def decode_step(self, st: DecodeState, token: int) -> np.ndarray:
        """Run one position (st.pos) for `token`; return its logits [V]."""
        t = st.pos
        h = self.w("tok_emb")[int(token)].copy()                      # [d]
        cos, sin = rope_cos_sin([t], self.hd, self.shape.rope_base)
        cos, sin = cos[0], sin[0]
        G = self.H // self.KV
        for l in range(self.L):
            p = f"{l}."
            a = rms_norm(h, self.w(p + "attn_norm"), self.eps)
            q = (self.w(p + "wq") @ a).reshape(self.H, self.hd)
            k = (self.w(p + "wk") @ a).reshape(self.KV, self.hd)
            v = (self.w(p + "wv") @ a).reshape(self.KV, self.hd)
            q = apply_rope(q, cos, sin)
            st.k[l].append(self._kv_round(apply_rope(k, cos, sin)))
            st.v[l].append(self._kv_round(v))
            Kc = np.stack(st.k[l])                                    # [t+1, KV, hd]
            Vc = np.stack(st.v[l])
            o = np.empty((self.H, self.hd), dtype=self.dtype)
            for hh in range(self.H):
                j = hh // G
                o[hh] = attention_one_query(q[hh], Kc[:, j, :], Vc[:, j, :])
            h = h + self.w(p + "wo") @ o.reshape(-1)
            b = rms_norm(h, self.w(p + "ffn_norm"), self.eps)
            g = self.w(p + "w_gate") @ b
            u = self.w(p + "w_up") @ b
            h = h + self.w(p + "w_down") @ (silu(g) * u)
        st.pos = t + 1
        hn = rms_norm(h, self.w("final_norm"), self.eps)
        return self.w("lm_head") @ hn

    def prefill(self, st: DecodeState, prompt: Sequence[int]) -> np.ndarray:
        """Feed the prompt one position at a time; logits of the last one."""
        logits = None
        for tok in prompt:
            logits = self.decode_step(st, int(tok))
        return logits

    def prefill_batched(self, prompt: Sequence[int]) -> Tuple[DecodeState, np.ndarray]:
        """Same state as `prefill`, with the prompt's K/V from one batched pass.

        The cache entries are the full-sequence path's K/V (causality makes
        them equal to the incremental ones); the last position's logits come
        from the same pass.
        """
        toks = np.asarray(prompt, dtype=np.int64)
        T = toks.shape[0]
        st = self.new_state()
        h = self.w("tok_emb")[toks]
        cos, sin = rope_cos_sin(range(T), self.hd, self.shape.rope_base)
        cos, sin = cos[:, None, :], sin[:, None, :]
        for l in range(self.L):
            p = f"{l}."
            a = rms_norm(h, self.w(p + "attn_norm"), self.eps)
            q = (a @ self.w(p + "wq").T).reshape(T, self.H, self.hd)
            k = (a @ self.w(p + "wk").T).reshape(T, self.KV, self.hd)
            v = (a @ self.w(p + "wv").T).reshape(T, self.KV, self.hd)
            q = apply_rope(q, cos, sin)
            k = self._kv_round(apply_rope(k, cos, sin))
            v = self._kv_round(v)
            st.k[l] = [k[i] for i in range(T)]
            st.v[l] = [v[i] for i in range(T)]
            o = causal_attention(q, k, v).reshape(T, self.H * self.hd)
            h = h + o @ self.w(p + "wo").T
            b = rms_norm(h, self.w(p + "ffn_norm"), self.eps)
            g = b @ self.w(p + "w_gate").T
            u = b @ self.w(p + "w_up").T
            h = h + (silu(g) * u) @ self.w(p + "w_down").T
        st.pos = T
        hn = rms_norm(h[-1], self.w("final_norm"), self.eps)
        return st, self.w("lm_head") @ hn

    def greedy(self, prompt: Sequence[int], n_steps: int, eos_id: int = -1,
               batched_prefill: bool = False):
        """Prefill then `n_steps` greedy decode steps.

        Returns (ids, logits): ids[0] = g0 picked after the prompt, ids[i]
        (i >= 1) picked by decode step i-1 (which fed ids[i-1] at position
        P+i-1); logits[i] are the logits ids[i] was picked from.  Stops after
        emitting `eos_id` when it is >= 0.
        """
        if batched_prefill:
            st, lg = self.prefill_batched(prompt)
        else:
            st = self.new_state()
            lg = self.prefill(st, prompt)
        ids = [argmax_lowest(lg)]
        logits = [lg]
        for _ in range(n_steps):
            if eos_id >= 0 and ids[-1] == eos_id:
                break
            lg = self.decode_step(st, ids[-1])
            ids.append(argmax_lowest(lg))
            logits.append(lg)
        return ids, np.stack(logits)

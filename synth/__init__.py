"""Seeded synthetic inputs for the batch-1 decode path: model shapes, weights,
prompts and forced token streams.

This module holds no arithmetic of the transformer itself.  It only draws
numbers, so that the CUDA path and the CPU oracle can be fed the very same
host fp16 buffers.  Every draw is a pure function of (seed, tensor index,
block index), independent of thread count and call order.

Recipe (applies to every model below):
  * weights: N(0, 1) drawn in fp32, scaled by 0.02, rounded to fp16 (RNE);
  * RMSNorm gains: exactly 1.0 (not drawn);
  * tensor order (its index selects the stream): tok_emb, then for each
    layer attn_norm, wq, wk, wv, wo, ffn_norm, w_gate, w_up, w_down, then
    final_norm, lm_head;
  * prompt ids: uniform in [0, vocab) from the stream seeded (seed + 1);
  * forced decode ids (teacher forcing): uniform in [0, vocab) from the
    stream seeded (seed + 2).

The pages measure a ~2B fp16 model ("Laneformer 2B") whose weights are not
available; the 28-layer d=2560 shapes below stand in for it at the same
scale, with random weights (revietech.ru, "Kog выжимает максимум из GPU:
3000 токенов/с", section "Модель Laneformer 2B").
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "ModelShape", "Workload", "WORKLOADS", "SynthModel", "make_model",
    "make_prompt", "make_forced_ids", "tensor_names", "WEIGHT_STD", "PROFILE_WORKLOADS",
    "workload",
]

WEIGHT_STD = 0.02
_BLOCK = 1 << 22          # elements per independently seeded block


@dataclasses.dataclass(frozen=True)
class ModelShape:
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    vocab: int
    rope_base: float = 10000.0
    rms_eps: float = 1e-5

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def n_params(self) -> int:
        d, L = self.d_model, self.n_layers
        per_layer = (d * self.q_dim + 2 * d * self.kv_dim + self.q_dim * d
                     + 3 * d * self.ffn_dim + 2 * d)
        return L * per_layer + 2 * self.vocab * d + d

    def matrix_bytes_per_token(self) -> int:
        """fp16 bytes of every weight matrix + norm gains + one embedding row."""
        d, L = self.d_model, self.n_layers
        per_layer = (d * self.q_dim + 2 * d * self.kv_dim + self.q_dim * d
                     + 3 * d * self.ffn_dim + 2 * d)
        return 2 * (L * per_layer + self.vocab * d + d + d)

    def kv_bytes_per_position(self) -> int:
        """fp16 K and V bytes of one position over all layers."""
        return 2 * self.n_layers * self.kv_dim * 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: ModelShape
    prompt_len: int
    decode_steps: int
    seed: int = 0

    @property
    def max_seq(self) -> int:
        return self.prompt_len + self.decode_steps

    def bytes_per_token_mean(self) -> float:
        """Algorithmic HBM bytes of one decode step at the mean position.

        Step i (0-based) runs at position P+i and reads K/V of positions
        0..P+i (P+i+1 of them) and writes one position.
        """
        s = self.shape
        mean_read_positions = self.prompt_len + (self.decode_steps + 1) / 2.0
        kv = s.kv_bytes_per_position() * (mean_read_positions + 1)
        return s.matrix_bytes_per_token() + kv


# The five workloads of the batch-1 decode benchmark, named by their shapes.
WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("tiny-l2-d256", ModelShape(2, 256, 4, 4, 64, 768, 2048), 16, 32),
    Workload("l16-d1024", ModelShape(16, 1024, 16, 4, 64, 2816, 32000), 128, 256),
    Workload("l28-d2560", ModelShape(28, 2560, 20, 4, 128, 6912, 50304), 512, 1024),
    Workload("l28-d2560-ctx8k", ModelShape(28, 2560, 20, 4, 128, 6912, 50304), 8192, 512),
    Workload("l32-d4096", ModelShape(32, 4096, 32, 8, 128, 14336, 128256,
                                     rope_base=500000.0), 1024, 512),
]}


# Smaller cases with the 2.2B model's per-layer shapes, for profiler captures
# (an ncu capture replays each launch dozens of times; these keep the device
# footprint to a couple of GB).
PROFILE_WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("l4-d2560", ModelShape(4, 2560, 20, 4, 128, 6912, 50304), 512, 8),
]}


def workload(name: str) -> Workload:
    return WORKLOADS[name] if name in WORKLOADS else PROFILE_WORKLOADS[name]


def tensor_names(n_layers: int) -> List[str]:
    """Fixed tensor order; the position of a name is its stream index."""
    names = ["tok_emb"]
    for l in range(n_layers):
        names += [f"{l}.{n}" for n in ("attn_norm", "wq", "wk", "wv", "wo",
                                       "ffn_norm", "w_gate", "w_up", "w_down")]
    names += ["final_norm", "lm_head"]
    return names


def _shape_of(name: str, s: ModelShape):
    d = s.d_model
    base = name.split(".")[-1]
    return {
        "tok_emb": (s.vocab, d), "lm_head": (s.vocab, d),
        "attn_norm": (d,), "ffn_norm": (d,), "final_norm": (d,),
        "wq": (s.q_dim, d), "wk": (s.kv_dim, d), "wv": (s.kv_dim, d),
        "wo": (d, s.q_dim), "w_gate": (s.ffn_dim, d), "w_up": (s.ffn_dim, d),
        "w_down": (d, s.ffn_dim),
    }[base]


def _fill_block(out_flat: np.ndarray, seed: int, tidx: int, b: int) -> None:
    lo = b * _BLOCK
    hi = min(out_flat.size, lo + _BLOCK)
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tidx, b])))
    v = rng.standard_normal(hi - lo, dtype=np.float32)
    v *= np.float32(WEIGHT_STD)
    out_flat[lo:hi] = v.astype(np.float16)


@dataclasses.dataclass
class SynthModel:
    shape: ModelShape
    seed: int
    tensors: Dict[str, np.ndarray]

    def layer(self, l: int) -> Dict[str, np.ndarray]:
        p = f"{l}."
        return {k[len(p):]: v for k, v in self.tensors.items() if k.startswith(p)}

    def __getitem__(self, name: str) -> np.ndarray:
        return self.tensors[name]


def make_model(shape: ModelShape, seed: int = 0, threads: Optional[int] = None,
               overrides: Optional[Dict[str, np.ndarray]] = None) -> SynthModel:
    """Draw every tensor of `shape` from `seed` (see the module recipe)."""
    names = tensor_names(shape.n_layers)
    tensors: Dict[str, np.ndarray] = {}
    jobs = []
    for tidx, name in enumerate(names):
        shp = _shape_of(name, shape)
        if name.endswith("norm"):
            tensors[name] = np.ones(shp, dtype=np.float16)
            continue
        arr = np.empty(shp, dtype=np.float16)
        tensors[name] = arr
        flat = arr.reshape(-1)
        nblk = (flat.size + _BLOCK - 1) // _BLOCK
        jobs += [(flat, tidx, b) for b in range(nblk)]
    threads = threads or min(32, os.cpu_count() or 1)
    if threads <= 1 or len(jobs) <= 1:
        for j in jobs:
            _fill_block(j[0], seed, j[1], j[2])
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda j: _fill_block(j[0], seed, j[1], j[2]), jobs))
    if overrides:
        for k, v in overrides.items():
            assert tensors[k].shape == v.shape, (k, v.shape)
            tensors[k] = np.ascontiguousarray(v, dtype=np.float16)
    return SynthModel(shape, seed, tensors)


def make_prompt(vocab: int, n: int, seed: int = 0) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed + 1, 0])))
    return rng.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


def make_forced_ids(vocab: int, n: int, seed: int = 0) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed + 2, 0])))
    return rng.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)

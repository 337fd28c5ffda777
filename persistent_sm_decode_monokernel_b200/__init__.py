"""Batch-1 decode monokernel for B200 (sm_100a).

The compute path is libkie.so (CUDA, C ABI in include/kie.h).  This package
holds its ctypes binding (`_kie`, same names as the C calls) and `Session`,
a convenience owner of the device buffers: PyTorch allocates device memory
and provides the stream, nothing more.
"""
from __future__ import annotations

from typing import Mapping, Optional, Sequence

import numpy as np

from . import _kie
from ._kie import (KieError, kie_check_desc, kie_create, kie_decode, kie_decode_forced,  # noqa: F401
                   kie_destroy, kie_get_stats, kie_kv_cache_bytes, kie_last_error,
                   kie_plan_units, kie_prefill, kie_rewind, kie_set_eos_ids,
                   kie_set_logits_capture, kie_set_option, kie_set_sampling,
                   kie_set_sampling_filter, kie_set_trace,
                   load_library, make_desc)

TRACE_PER_LAYER = 24   # trace slots per layer (kie.h, kie_set_trace)

__all__ = ["TRACE_PER_LAYER", "Session", "KieError", "load_library", "make_desc", "upload_weights"]


def upload_weights(host: Mapping[str, np.ndarray], device="cuda"):
    """Copies host fp16 arrays to device tensors (same names)."""
    import torch
    out = {}
    for k, v in host.items():
        out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(device)
    return out


class Session:
    """One decode session on the current CUDA device.

    shape: any object with n_layers, d_model, n_heads, n_kv_heads, head_dim,
    ffn_dim, vocab, rope_base, rms_eps.  weights: device fp16 tensors named
    tok_emb, final_norm, lm_head and "{l}.{attn_norm,wq,wk,wv,wo,ffn_norm,
    w_gate,w_up,w_down}".  The KV cache is allocated here with torch.

    kie_create keeps its own packed copy of every weight matrix and from
    then on reads only tok_emb and the norm gains of `weights`.  With
    keep_matrices=False the session drops its references to the matrices
    right after kie_create (their memory is freed once the caller drops
    its own), which halves the weights' device footprint; re-planning the
    chunk size (KIE_OPT_CHUNK_BYTES) or the weight format then raises, since
    it re-reads them.

    weight_format: "fp16" (the caller's weights as they are) or "fp8" (the
    packed stream holds FP8 E4M3 codes with one fp32 scale per row,
    KIE_OPT_WEIGHT_FP8), set before the matrices are released.
    """

    # the tensors kie_create's packed copy does not replace
    _KEPT = ("tok_emb", "final_norm")

    def __init__(self, shape, weights: Mapping[str, object], max_seq: int, eos_id: int = -1,
                 stream=None, keep_matrices: bool = True, weight_format: str = "fp16"):
        import torch
        load_library()
        self.shape = shape
        self.desc = make_desc(shape.n_layers, shape.d_model, shape.n_heads, shape.n_kv_heads,
                              shape.head_dim, shape.ffn_dim, shape.vocab, shape.rope_base,
                              shape.rms_eps, max_seq, eos_id)
        st = kie_check_desc(self.desc)
        if st != _kie.KIE_OK:
            raise KieError(st, "kie_check_desc")
        nbytes = kie_kv_cache_bytes(self.desc)
        self.kv = torch.empty(nbytes // 2, dtype=torch.float16, device="cuda")
        self.weights = weights
        if stream is None:
            stream = torch.cuda.current_stream()
        self.stream = stream
        self.ctx = kie_create(self.desc, weights, self.kv, stream.cuda_stream)
        self._capture = None
        if weight_format not in ("fp16", "fp8"):
            raise ValueError(f"weight_format {weight_format!r}: 'fp16' or 'fp8'")
        if weight_format == "fp8":
            kie_set_option(self.ctx, _kie.KIE_OPT_WEIGHT_FP8, 1)
        if not keep_matrices:
            self.release_matrices()

    def release_matrices(self) -> None:
        """Drops this session's references to the weight matrices (kept:
        the embedding and the norm gains, which the kernel still reads).
        The batched prefill reads the matrices, so prefill then runs every
        position as a decode step."""
        kie_set_option(self.ctx, _kie.KIE_OPT_BATCHED_PREFILL, 0)
        self.weights = {k: v for k, v in self.weights.items()
                        if k in self._KEPT or k.endswith("norm")}
        self._matrices_released = True

    def prefill(self, ids: Sequence[int]) -> int:
        return kie_prefill(self.ctx, ids)

    def decode(self, n_steps: int, out: Optional[np.ndarray] = None) -> np.ndarray:
        return kie_decode(self.ctx, n_steps, out)

    def decode_forced(self, ids: Sequence[int]) -> np.ndarray:
        return kie_decode_forced(self.ctx, ids)

    def rewind(self, pos: int) -> None:
        kie_rewind(self.ctx, pos)

    def capture_logits(self, rows: int):
        """Turns logit capture on into a fresh [rows, vocab] fp32 device tensor."""
        import torch
        self._capture = torch.empty((rows, self.shape.vocab), dtype=torch.float32, device="cuda")
        kie_set_logits_capture(self.ctx, self._capture, rows)
        return self._capture

    def capture_off(self) -> None:
        kie_set_logits_capture(self.ctx, None, 0)
        self._capture = None

    def trace(self, steps: int, cta: int = 0):
        """Turns the stage trace on for `steps` steps of CTA `cta`; returns the
        [steps, n_layers*24 + 4] int64 device buffer it fills.  cta=-1 traces
        every CTA into a [steps, grid, n_layers*24 + 4] buffer."""
        import torch
        per = self.shape.n_layers * TRACE_PER_LAYER + 4
        shape = (steps, per) if cta >= 0 else (steps, self.stats()["grid"], per)
        self._trace = torch.zeros(shape, dtype=torch.int64, device="cuda")
        kie_set_trace(self.ctx, self._trace, self._trace.numel(), cta)
        return self._trace

    def trace_off(self) -> None:
        kie_set_trace(self.ctx, None, 0, 0)
        self._trace = None

    def set_option(self, opt: int, value: int) -> None:
        rereads = opt in (_kie.KIE_OPT_CHUNK_BYTES, _kie.KIE_OPT_WEIGHT_FP8) or (
            opt == _kie.KIE_OPT_BATCHED_PREFILL and value)
        if rereads and getattr(self, "_matrices_released", False):
            raise ValueError("this option re-reads the weight matrices, which this session "
                             "has released (keep_matrices=False)")
        kie_set_option(self.ctx, opt, value)

    def set_sampling(self, temperature: float, seed: int = 0, top_k: int = 0,
                     top_p: float = 1.0) -> None:
        """temperature 0 = greedy (default); > 0 samples in the kernel, from
        the top_k largest logits (0 = all) and of those the top_p nucleus
        (1 = all; top_p < 1 needs top_k >= 1)."""
        kie_set_sampling(self.ctx, temperature, seed)
        kie_set_sampling_filter(self.ctx, top_k, top_p)

    def set_eos_ids(self, ids: Sequence[int]) -> None:
        """Ids that end a decode ([] = the descriptor's eos_id)."""
        kie_set_eos_ids(self.ctx, ids)

    def stats(self):
        return kie_get_stats(self.ctx)

    def close(self) -> None:
        if getattr(self, "ctx", None):
            kie_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

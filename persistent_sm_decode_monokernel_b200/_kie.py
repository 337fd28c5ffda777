"""ctypes binding of libkie.so (include/kie.h): argument marshalling only.

Every step of the decode path runs in the CUDA library; this module only
turns Python/torch arguments into the C ABI's pointers and sizes.  There is
no fallback: if libkie.so is missing or fails to load, importing the
binding raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Mapping, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkie.so")

# ---- status codes and options (kie.h)
KIE_OK = 0
KIE_ERR_INVALID_ARG = 1
KIE_ERR_UNSUPPORTED = 2
KIE_ERR_CUDA = 3
KIE_ERR_CAPACITY = 4
KIE_ERR_STATE = 5
KIE_ERR_TIMEOUT = 6
KIE_ERR_PROTOCOL = 7
KIE_ERR_TOO_LARGE = 8
KIE_ERR_HOST_MEMORY = 9

KIE_NOALLOC_MAX_WEIGHT_BYTES = 16 * 1024 * 1024
KIE_MAX_EOS_IDS = 8
KIE_MAX_TOP_K = 64

KIE_OPT_TIMEOUT_NS = 1
KIE_OPT_CHUNK_BYTES = 2
KIE_OPT_MIN_SPLIT_LEN = 3
KIE_OPT_FAULT_CTA = 4
KIE_OPT_FAULT_STEP = 5
KIE_OPT_FAULT_LAYER = 6
KIE_OPT_FAULT_STAGE = 7
KIE_OPT_POLL_BACKOFF_NS = 8
KIE_OPT_TRACE_CLOCK = 9
KIE_OPT_L2_PREFETCH_BYTES = 10
KIE_OPT_WEIGHT_FP8 = 11
KIE_OPT_BATCHED_PREFILL = 12
KIE_OPT_TMEM_PARK = 13

STAGE_QKV, STAGE_O, STAGE_GU, STAGE_DOWN, STAGE_LM = range(5)


class KieModelDesc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn_dim", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("rope_base", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("max_seq", ctypes.c_int32),
                ("eos_id", ctypes.c_int32)]


class KieLayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")]


class KieWeights(ctypes.Structure):
    _fields_ = [("tok_emb", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("lm_head", ctypes.c_void_p), ("layers", ctypes.POINTER(KieLayerWeights))]


class KieStats(ctypes.Structure):
    _fields_ = [("pos", ctypes.c_int32), ("grid", ctypes.c_int32),
                ("ring_bytes", ctypes.c_int32), ("chunk_bytes", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("last_steps", ctypes.c_int32),
                ("last_device_ms", ctypes.c_float), ("launches", ctypes.c_uint64),
                ("loop_cycles", ctypes.c_double), ("sync_wait_cycles", ctypes.c_double),
                ("stream_wait_cycles", ctypes.c_double), ("producer_wait_cycles", ctypes.c_double),
                ("sync_wait_max_frac", ctypes.c_double), ("last_prefill_ms", ctypes.c_double),
                ("last_prefill_batched", ctypes.c_int32)]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_PI32 = ctypes.POINTER(ctypes.c_int32)
_PDESC = ctypes.POINTER(KieModelDesc)

# name -> (restype, argtypes); the exported symbols of kie.h
SIGNATURES = {
    "kie_kv_cache_bytes": (ctypes.c_size_t, [_PDESC]),
    "kie_check_desc": (ctypes.c_int, [_PDESC]),
    "kie_create": (ctypes.c_int, [_PDESC, ctypes.POINTER(KieWeights), _P, _P,
                                  ctypes.POINTER(ctypes.c_void_p)]),
    "kie_prefill": (ctypes.c_int, [_P, _PI32, _I32, _PI32]),
    "kie_decode": (ctypes.c_int, [_P, _I32, _PI32, _PI32]),
    "kie_decode_forced": (ctypes.c_int, [_P, _PI32, _I32, _PI32]),
    "kie_rewind": (ctypes.c_int, [_P, _I32]),
    "kie_set_logits_capture": (ctypes.c_int, [_P, _P, _I32]),
    "kie_set_option": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int64]),
    "kie_set_sampling": (ctypes.c_int, [_P, ctypes.c_float, ctypes.c_uint64]),
    "kie_set_eos_ids": (ctypes.c_int, [_P, _PI32, _I32]),
    "kie_set_trace": (ctypes.c_int, [_P, _P, _I32, _I32]),
    "kie_get_stats": (ctypes.c_int, [_P, ctypes.POINTER(KieStats)]),
    "kie_status_str": (ctypes.c_char_p, [ctypes.c_int]),
    "kie_last_error": (ctypes.c_char_p, [_P]),
    "kie_destroy": (ctypes.c_int, [_P]),
    "kie_plan_units": (ctypes.c_int, [_PDESC, _I32, _I32, _I32, _PI32, _PI32]),
    "kie_plan_gemv_work": (ctypes.c_int, [_PDESC, _I32, _I32, _I32, _I32, _I32, _PI32]),
    "kie_gemv_f16": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P,
                                    ctypes.POINTER(ctypes.c_float),
                                    ctypes.POINTER(ctypes.c_double)]),
    "kie_gemv_f16_noalloc": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _P]),
    "kie_set_sampling_filter": (ctypes.c_int, [_P, _I32, ctypes.c_float]),
    "kie_quantize_e4m3": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _P]),
}

_lib: Optional[ctypes.CDLL] = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libkie.so (built by `build.py`); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m persistent_sm_decode_monokernel_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class KieError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        lib = load_library()
        self.status = status
        msg = f"{where}: {lib.kie_status_str(status).decode()}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


def _check(st: int, where: str, ctx=None) -> None:
    if st != KIE_OK:
        detail = ""
        if ctx:
            detail = (load_library().kie_last_error(ctx) or b"").decode()
        raise KieError(st, where, detail)


def make_desc(n_layers: int, d_model: int, n_heads: int, n_kv_heads: int, head_dim: int,
              ffn_dim: int, vocab: int, rope_base: float, rms_eps: float, max_seq: int,
              eos_id: int = -1) -> KieModelDesc:
    return KieModelDesc(n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn_dim, vocab,
                        rope_base, rms_eps, max_seq, eos_id)


def kie_kv_cache_bytes(desc: KieModelDesc) -> int:
    return int(load_library().kie_kv_cache_bytes(ctypes.byref(desc)))


def kie_check_desc(desc: Optional[KieModelDesc]) -> int:
    return int(load_library().kie_check_desc(ctypes.byref(desc) if desc is not None else None))


def kie_plan_units(desc: KieModelDesc, grid: int, stage: int, cta: int):
    b, e = ctypes.c_int32(), ctypes.c_int32()
    _check(load_library().kie_plan_units(ctypes.byref(desc), grid, stage, cta,
                                         ctypes.byref(b), ctypes.byref(e)), "kie_plan_units")
    return b.value, e.value


def kie_plan_gemv_work(desc: KieModelDesc, grid: int, stage: int, cta: int,
                       chunk_bytes: int = 32768, fp8: int = 0):
    """(rows, pieces per row, rows per block, parts per row, blocks, result
    slots) of CTA `cta`'s GEMV work in `stage` (see kie.h)."""
    out = (ctypes.c_int32 * 6)()
    _check(load_library().kie_plan_gemv_work(ctypes.byref(desc), grid, stage, cta, chunk_bytes,
                                             fp8, out), "kie_plan_gemv_work")
    return tuple(int(v) for v in out)


LAYER_NAMES = ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")


def _ptr(t) -> int:
    return int(t.data_ptr())


def weights_struct(weights: Mapping[str, object], n_layers: int):
    """kie_weights from device tensors named tok_emb, final_norm, lm_head and
    "{layer}.{attn_norm,wq,wk,wv,wo,ffn_norm,w_gate,w_up,w_down}"."""
    layers = (KieLayerWeights * n_layers)()
    for l in range(n_layers):
        for n in LAYER_NAMES:
            setattr(layers[l], n, _ptr(weights[f"{l}.{n}"]))
    w = KieWeights(_ptr(weights["tok_emb"]), _ptr(weights["final_norm"]),
                   _ptr(weights["lm_head"]), layers)
    return w, layers


def kie_create(desc: KieModelDesc, weights: Mapping[str, object], kv_cache, stream=None):
    """Returns an opaque context handle (int)."""
    lib = load_library()
    w, keep = weights_struct(weights, desc.n_layers)
    ctx = ctypes.c_void_p()
    st = lib.kie_create(ctypes.byref(desc), ctypes.byref(w), _ptr(kv_cache),
                        ctypes.c_void_p(stream or 0), ctypes.byref(ctx))
    _check(st, "kie_create")
    return ctx.value


def kie_prefill(ctx, ids: Sequence[int]) -> int:
    a = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    first = ctypes.c_int32()
    _check(load_library().kie_prefill(ctx, a.ctypes.data_as(_PI32), a.size, ctypes.byref(first)),
           "kie_prefill", ctx)
    return first.value


def kie_decode(ctx, n_steps: int, out: Optional[np.ndarray] = None) -> np.ndarray:
    """Decode of n_steps ids in one launch; returns the ids written."""
    if out is None:
        out = np.empty(max(n_steps, 1), dtype=np.int32)
    n_out = ctypes.c_int32()
    _check(load_library().kie_decode(ctx, n_steps, out.ctypes.data_as(_PI32), ctypes.byref(n_out)),
           "kie_decode", ctx)
    return out[:n_out.value]


def kie_decode_forced(ctx, ids: Sequence[int]) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    out = np.empty(max(a.size, 1), dtype=np.int32)
    _check(load_library().kie_decode_forced(ctx, a.ctypes.data_as(_PI32), a.size,
                                            out.ctypes.data_as(_PI32)), "kie_decode_forced", ctx)
    return out[:a.size]


def kie_rewind(ctx, pos: int) -> None:
    _check(load_library().kie_rewind(ctx, pos), "kie_rewind", ctx)


def kie_set_logits_capture(ctx, logits=None, rows: int = 0) -> None:
    ptr = _ptr(logits) if logits is not None else None
    _check(load_library().kie_set_logits_capture(ctx, ptr, rows if logits is not None else 0),
           "kie_set_logits_capture", ctx)


def kie_set_trace(ctx, buf=None, capacity: int = 0, cta: int = 0) -> None:
    ptr = _ptr(buf) if buf is not None else None
    _check(load_library().kie_set_trace(ctx, ptr, capacity if buf is not None else 0, cta),
           "kie_set_trace", ctx)


def kie_set_option(ctx, opt: int, value: int) -> None:
    _check(load_library().kie_set_option(ctx, opt, int(value)), "kie_set_option", ctx)


def kie_set_sampling(ctx, temperature: float, seed: int = 0) -> None:
    """temperature 0 = greedy; > 0 = in-kernel temperature sampling."""
    _check(load_library().kie_set_sampling(ctx, float(temperature), int(seed) & ((1 << 64) - 1)),
           "kie_set_sampling", ctx)


def kie_set_sampling_filter(ctx, top_k: int = 0, top_p: float = 1.0) -> None:
    """Restricts sampled draws to the top_k largest logits, then to the
    top_p nucleus of those (0 and 1: off)."""
    _check(load_library().kie_set_sampling_filter(ctx, int(top_k), float(top_p)),
           "kie_set_sampling_filter", ctx)


def kie_set_eos_ids(ctx, ids: Sequence[int]) -> None:
    a = np.ascontiguousarray(np.asarray(list(ids), dtype=np.int32))
    _check(load_library().kie_set_eos_ids(ctx, a.ctypes.data_as(_PI32) if a.size else None,
                                          a.size), "kie_set_eos_ids", ctx)


def kie_get_stats(ctx) -> Dict[str, float]:
    s = KieStats()
    _check(load_library().kie_get_stats(ctx, ctypes.byref(s)), "kie_get_stats", ctx)
    return {f: getattr(s, f) for f, _ in KieStats._fields_}


def kie_last_error(ctx) -> str:
    return (load_library().kie_last_error(ctx) or b"").decode()


def kie_gemv_f16(W, x, y, iters: int = 1, mode: int = 1, chunk_bytes: int = 32768, stream=None):
    """y = W x with the decode kernel's GEMV engine; returns (ms, stats dict)."""
    N, K = W.shape
    ms = ctypes.c_float()
    st = (ctypes.c_double * 4)()
    _check(load_library().kie_gemv_f16(_ptr(W), _ptr(x), _ptr(y) if y is not None else None,
                                       N, K, iters, mode, chunk_bytes,
                                       ctypes.c_void_p(stream or 0), ctypes.byref(ms), st),
           "kie_gemv_f16")
    return ms.value, {"stream_wait_cycles": st[0], "producer_wait_cycles": st[1],
                      "grid": int(st[2]), "ring_bytes": int(st[3])}


def kie_quantize_e4m3(W, codes, scales, stream=None) -> None:
    """FP8 E4M3 codes [N, K] (uint8 tensor) and row scales [N] (fp32) of
    an fp16 matrix W [N, K]: the rule of KIE_OPT_WEIGHT_FP8 (see kie.h)."""
    N, K = W.shape
    _check(load_library().kie_quantize_e4m3(_ptr(W), N, K, _ptr(codes), _ptr(scales),
                                            ctypes.c_void_p(stream or 0)), "kie_quantize_e4m3")


def kie_gemv_f16_noalloc(W, x, y, stream=None) -> None:
    """y = W x through the entry point that allocates no device memory (its
    scratch is a fixed array inside the library; see kie.h)."""
    N, K = W.shape
    _check(load_library().kie_gemv_f16_noalloc(_ptr(W), _ptr(x), _ptr(y), N, K,
                                               ctypes.c_void_p(stream or 0)),
           "kie_gemv_f16_noalloc")


def kie_destroy(ctx) -> None:
    if ctx:
        _check(load_library().kie_destroy(ctx), "kie_destroy")

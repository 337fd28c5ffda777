"""FP8 weight quantisation of the decode path -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this module; the library never does.  It shares no code with the CUDA
path.

The pages put FP8 quantisation on the roadmap of the decode engine without
naming a format, a scale granularity or where the scales are applied
(revietech.ru, "Kog выжимает максимум из GPU: 3000 токенов/с", section
"Ограничения подхода").  The reading taken here is the plainest one that
keeps the rest of the path unchanged:

  * format: FP8 E4M3 in its "fn" form -- 1 sign bit, 4 exponent bits with
    bias 7, 3 mantissa bits; no infinities; the codes S.1111.111 are NaN, so
    the largest finite magnitude is 1.75 * 2^8 = 448; exponent field 0 holds
    the subnormals M/8 * 2^-6;
  * granularity: one fp32 scale per output row of every weight matrix
    (Wq, Wk, Wv, Wo, W_gate, W_up, W_down and the LM head; the embedding
    table and the norm gains stay fp16):
        s_r = max_c |W_rc| / 448          (fp32 division; s_r = 1 for a zero row)
        q_rc = E4M3(W_rc / s_r)            (fp32 division, round to nearest,
                                            ties to the even code, magnitudes
                                            beyond 448 saturate to 448)
  * the quantised model is the same transformer with W_rc replaced by
    s_r * value(q_rc); a matrix-vector product is y_r = s_r * sum_c value(q_rc) x_c.

Functions: `e4m3_value` (code -> value, from the bit fields), `e4m3_encode`
(value -> code, nearest finite value by search over the 127 non-negative
finite values), `row_scales`, `quantize_rows`, `dequantize_rows`,
`quantized_matvec`, and `fp8_model`, which returns the model whose matrices
are the dequantised weights (to feed `OracleModel` unchanged).
Pinned by tests/test_oracle_fp8.py.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = ["E4M3_MAX", "FP8_MATRICES", "e4m3_value", "e4m3_encode", "row_scales",
           "quantize_rows", "dequantize_rows", "quantized_matvec", "fp8_model",
           "fp8_matrix_names"]

E4M3_MAX = 448.0
EXP_BIAS = 7
# the weight matrices that are stored in FP8 (per-layer names, then the head)
FP8_MATRICES = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")


def e4m3_value(codes) -> np.ndarray:
    """Value of each E4M3 code (uint8 array) as float64; NaN for S.1111.111."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - EXP_BIAS).astype(np.int64))
    sub = sign * np.ldexp(m / 8.0, 1 - EXP_BIAS)
    v = np.where(e == 0, sub, normal)
    return np.where((e == 0xF) & (m == 0x7), np.nan, v)


# the 127 non-negative finite values, increasing with the code 0 .. 126
_POS = e4m3_value(np.arange(127, dtype=np.uint8))
# value of every code, looked up by dequantize_rows
_VALUES = e4m3_value(np.arange(256, dtype=np.uint8))


def e4m3_encode(x) -> np.ndarray:
    """E4M3 code (uint8) of each value: the nearest finite value, ties to the
    even code (mantissa LSB 0), magnitudes beyond 448 saturated to 448; the
    sign bit is the sign of x (so -0.0 and negatives that round to zero get
    code 0x80).  Large arrays go through in blocks (the same arithmetic)."""
    x = np.asarray(x)
    if x.size > _BLOCK:
        flat = x.reshape(-1)
        out = np.empty(flat.shape, dtype=np.uint8)

        def block(i):
            out[i:i + _BLOCK] = _encode_block(flat[i:i + _BLOCK])
        with ThreadPoolExecutor(min(32, os.cpu_count() or 1)) as ex:
            list(ex.map(block, range(0, flat.size, _BLOCK)))
        return out.reshape(x.shape)
    return _encode_block(x)


_BLOCK = 1 << 20


def _encode_block(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_POS, a, side="left")            # first value >= a
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(np.signbit(x), code | np.uint8(0x80), code)
    return code.astype(np.uint8)


def row_scales(W) -> np.ndarray:
    """fp32 s_r = max_c |W_rc| / 448 per row (1 for a zero row)."""
    W = np.asarray(W, dtype=np.float32)
    amax = np.max(np.abs(W), axis=1)
    s = amax / np.float32(E4M3_MAX)
    return np.where(amax > 0, s, np.float32(1.0)).astype(np.float32)


def quantize_rows(W):
    """(codes uint8 [N, K], scales fp32 [N]) of an fp16 / fp32 matrix W [N, K];
    W_rc / s_r is formed in fp32."""
    W32 = np.asarray(W, dtype=np.float32)
    s = row_scales(W32)
    return e4m3_encode(W32 / s[:, None]), s


def dequantize_rows(codes, scales, dtype=np.float64) -> np.ndarray:
    """s_r * value(q_rc) in `dtype`."""
    v = _VALUES.astype(dtype)[np.asarray(codes, dtype=np.uint8)]
    return v * np.asarray(scales, dtype=dtype)[:, None]


def quantized_matvec(codes, scales, x) -> np.ndarray:
    """y_r = s_r * sum_c value(q_rc) x_c, in float64."""
    v = e4m3_value(codes)
    return np.asarray(scales, dtype=np.float64) * (v @ np.asarray(x, dtype=np.float64))


def fp8_matrix_names(n_layers: int):
    """Names (synth tensor names) of every matrix stored in FP8."""
    return [f"{l}.{n}" for l in range(n_layers) for n in FP8_MATRICES] + ["lm_head"]


class _Model:
    def __init__(self, shape, seed, tensors):
        self.shape, self.seed, self.tensors = shape, seed, tensors

    def __getitem__(self, name):
        return self.tensors[name]


def fp8_model(model, dtype=np.float32):
    """The model whose FP8 matrices are replaced by their dequantised values
    (in `dtype`); the embedding table and the norm gains are kept.  Returns
    (model, {name: (codes, scales)})."""
    tensors = dict(model.tensors)
    q = {}
    for name in fp8_matrix_names(model.shape.n_layers):
        codes, s = quantize_rows(model.tensors[name])
        q[name] = (codes, s)
        tensors[name] = dequantize_rows(codes, s, dtype=dtype)
    return _Model(model.shape, getattr(model, "seed", 0), tensors), q

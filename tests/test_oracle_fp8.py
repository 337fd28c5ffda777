"""Pins of the FP8 (E4M3, per-row scale) oracle to things other than itself:
the format's closed-form values, two library implementations of E4M3 (torch's
float8_e4m3fn and ml_dtypes' float8_e4m3fn), the round-to-nearest-even rule
at constructed midpoints, the quantisation error bound, and brute-force loops
for the quantised matrix-vector product and the quantised model."""
import math

import numpy as np
import pytest

import synth
from oracle import OracleModel
from oracle import fp8

# ------------------------------------------------------------ code <-> value


def test_e4m3_closed_form_values():
    v = fp8.e4m3_value
    assert v(0x38) == 1.0                      # E = 7, M = 0
    assert v(0x7E) == 448.0                    # E = 15, M = 6: the largest finite
    assert v(0x08) == 2.0 ** -6                # smallest normal
    assert v(0x01) == 2.0 ** -9                # smallest subnormal: 1/8 * 2^-6
    assert v(0x07) == 7 * 2.0 ** -9            # largest subnormal
    assert v(0x3C) == 1.5
    assert v(0xB8) == -1.0 and v(0xC0) == -2.0
    assert v(0x00) == 0.0 and math.copysign(1.0, v(0x80)) == -1.0
    assert math.isnan(v(0x7F)) and math.isnan(v(0xFF))
    assert np.sum(np.isnan(v(np.arange(256, dtype=np.uint8)))) == 2


def test_e4m3_values_match_torch_and_ml_dtypes():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    ours = fp8.e4m3_value(codes)
    t = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(ours, t)          # NaNs compare equal here
    ml = pytest.importorskip("ml_dtypes")
    m = codes.view(ml.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(ours, m)


def _library_codes(x):
    torch = pytest.importorskip("torch")
    return torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_on_random_and_midpoints():
    rng = np.random.default_rng(0)
    vals = fp8.e4m3_value(np.arange(127, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2                    # every tie inside the range
    x = np.concatenate([
        rng.standard_normal(20000) * 10 ** rng.uniform(-4, 2.5, 20000),
        mids, -mids, vals, -vals,
        np.nextafter(mids, 0), np.nextafter(mids, 1e9),
    ]).astype(np.float32)
    x = x[np.abs(x) <= 448]                              # torch overflows to NaN, we saturate
    np.testing.assert_array_equal(fp8.e4m3_encode(x), _library_codes(x))
    ml = pytest.importorskip("ml_dtypes")
    np.testing.assert_array_equal(fp8.e4m3_encode(x), x.astype(ml.float8_e4m3fn).view(np.uint8))


def test_e4m3_ties_go_to_the_even_code():
    enc = fp8.e4m3_encode
    assert enc(1.0625) == 0x38                 # 1.0 (M=0) vs 1.125 (M=1)
    assert enc(1.1875) == 0x3A                 # 1.125 (M=1) vs 1.25 (M=2)
    assert enc(1.9375) == 0x40                 # 1.875 (E7 M7) vs 2.0 (E8 M0)
    assert enc(2.0 ** -10) == 0x00             # 0 vs 2^-9
    assert enc(3 * 2.0 ** -10) == 0x02         # 2^-9 (M=1) vs 2 * 2^-9 (M=2)
    assert enc(464.0) == 0x7E                  # midpoint above 448 stays finite


def test_e4m3_saturates_and_round_trips():
    enc = fp8.e4m3_encode
    assert enc(449.0) == 0x7E and enc(1e6) == 0x7E and enc(-1e30) == 0xFE
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    np.testing.assert_array_equal(enc(fp8.e4m3_value(codes)), codes)


# ------------------------------------------------------------- quantisation


def test_row_scale_maps_each_row_max_to_448():
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((40, 96)) * 0.02).astype(np.float16)
    W[3] = 0
    codes, s = fp8.quantize_rows(W)
    assert s.dtype == np.float32 and s[3] == 1.0 and np.all(codes[3] & 0x7F == 0)
    amax = np.max(np.abs(W.astype(np.float32)), axis=1)
    np.testing.assert_array_equal(s[amax > 0], (amax / np.float32(448))[amax > 0])
    mags = codes & 0x7F
    for r in range(40):
        if r == 3:
            continue
        c = int(np.argmax(np.abs(W[r].astype(np.float32))))
        assert mags[r, c] == 0x7E, (r, mags[r, c])
        assert mags[r].max() == 0x7E


def test_quantisation_error_within_half_a_step():
    # |W - s q| <= s * (half the E4M3 spacing at |W|/s): 2^-4 relative for
    # normals, s * 2^-10 absolute below the smallest normal
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float16)
    codes, s = fp8.quantize_rows(W)
    Wd = fp8.dequantize_rows(codes, s)
    a = np.abs(W.astype(np.float64)) / s[:, None]
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    half = 2.0 ** (e - 4)                                # half of 2^(e-3)
    err = np.abs(W.astype(np.float64) - Wd) / s[:, None]
    assert np.all(err <= half * (1 + 1e-6) + 1e-12)
    rel = np.max(np.abs(W - Wd)) / np.max(np.abs(W))
    assert 1e-4 < rel < 0.07


def test_quantized_matvec_bruteforce():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((7, 33)) * 0.05).astype(np.float16)
    x = rng.standard_normal(33)
    codes, s = fp8.quantize_rows(W)
    want = []
    deq = np.empty((7, 33))
    for r in range(7):
        acc = 0.0
        for c in range(33):
            b = int(codes[r, c])
            sign = -1.0 if b & 0x80 else 1.0
            e, m = (b >> 3) & 15, b & 7
            val = sign * (m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
            deq[r, c] = float(s[r]) * val
            acc += val * x[c]
        want.append(float(s[r]) * acc)
    np.testing.assert_allclose(fp8.quantized_matvec(codes, s, x), want, rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(fp8.dequantize_rows(codes, s), deq)


def test_fp8_model_replaces_only_the_matrices():
    shp = synth.ModelShape(2, 64, 4, 2, 16, 96, 97)
    m = synth.make_model(shp, seed=3)
    q, codes = fp8.fp8_model(m, dtype=np.float64)
    assert set(codes) == set(fp8.fp8_matrix_names(2))
    for k, v in m.tensors.items():
        if k in codes:
            c, s = codes[k]
            np.testing.assert_array_equal(q[k], fp8.dequantize_rows(c, s))
            assert not np.array_equal(q[k], v.astype(np.float64))
        else:
            np.testing.assert_array_equal(q[k], v)
    toks = synth.make_prompt(97, 6, seed=3)
    a = OracleModel(m, dtype=np.float64).forward(toks)
    b = OracleModel(q, dtype=np.float64).forward(toks)
    rel = np.max(np.abs(a - b)) / np.max(np.abs(a))
    assert 1e-4 < rel < 0.2, rel


# ------------------------------------------------- planted mistakes (oracle)

def _value_bias8(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e, m = (c >> 3) & 0xF, c & 0x7
    v = np.where(e == 0, sign * np.ldexp(m / 8.0, -7), sign * np.ldexp(1.0 + m / 8.0, e - 8))
    return np.where((e == 0xF) & (m == 0x7), np.nan, v)


def _encode_ties_away(x):
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 448.0)
    hi = np.minimum(np.searchsorted(fp8._POS, a, side="left"), 126)
    lo = np.maximum(hi - 1, 0)
    code = np.where(fp8._POS[hi] - a <= a - fp8._POS[lo], hi, lo).astype(np.uint8)
    return np.where(np.signbit(x), code | np.uint8(0x80), code).astype(np.uint8)


def _encode_truncate(x):
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 448.0)
    code = np.maximum(np.searchsorted(fp8._POS, a, side="right") - 1, 0).astype(np.uint8)
    return np.where(np.signbit(x), code | np.uint8(0x80), code).astype(np.uint8)


def _encode_no_saturation(x):
    x = np.asarray(x, dtype=np.float64)
    out = fp8.__dict__["_orig_encode"](x)
    return np.where(np.abs(x) > 448, np.uint8(0x7F) | (out & 0x80), out).astype(np.uint8)


def _scales_fnuz_max(W):
    W = np.asarray(W, dtype=np.float32)
    amax = np.max(np.abs(W), axis=1)
    return np.where(amax > 0, amax / np.float32(240), np.float32(1)).astype(np.float32)


def _scales_per_tensor(W):
    W = np.asarray(W, dtype=np.float32)
    return np.full(W.shape[0], np.max(np.abs(W)) / np.float32(448), dtype=np.float32)


FP8_MUTATIONS = [
    ("e4m3_value", _value_bias8, test_e4m3_closed_form_values),
    ("e4m3_encode", _encode_ties_away, test_e4m3_ties_go_to_the_even_code),
    ("e4m3_encode", _encode_ties_away, test_e4m3_encode_matches_torch_on_random_and_midpoints),
    ("e4m3_encode", _encode_truncate, test_e4m3_encode_matches_torch_on_random_and_midpoints),
    ("e4m3_encode", _encode_no_saturation, test_e4m3_saturates_and_round_trips),
    ("row_scales", _scales_fnuz_max, test_row_scale_maps_each_row_max_to_448),
    ("row_scales", _scales_per_tensor, test_row_scale_maps_each_row_max_to_448),
]


@pytest.mark.parametrize("name,bad,pin", FP8_MUTATIONS,
                         ids=[f"{m[1].__name__}->{m[2].__name__}" for m in FP8_MUTATIONS])
def test_fp8_pin_catches_planted_mistake(monkeypatch, name, bad, pin):
    monkeypatch.setitem(fp8.__dict__, "_orig_encode", fp8.e4m3_encode)
    monkeypatch.setattr(fp8, name, bad)
    with pytest.raises(AssertionError):
        pin()

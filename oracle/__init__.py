"""Oracle for the batch-1 decode path -- TEST INFRASTRUCTURE.

A plain, slow CPU implementation (numpy, float32 or float64) of what the
decode monokernel computes, written from the definitions and sharing no code
with the CUDA path.  Only `tests/`, `__graft_entry__.smoke()` and the CPU
baseline leg of `bench.py` may import it; the library itself never does.

Every function carries its definition in its docstring; `tests/test_oracle_pins.py`
pins each of them to closed forms, invariants and brute force, and
`tests/test_oracle_sampling.py` pins the sampler (`oracle.sampling`) to
numpy's own Philox generator and to the softmax distribution it must draw,
and `tests/test_oracle_fp8.py` pins the FP8 weight quantisation
(`oracle.fp8`: E4M3 codes, per-row scales, the dequantised model) to the
format's closed forms, torch's and ml_dtypes' E4M3 conversions and brute
force.  Parity status
of each function: all pinned (none is "parity unpinned").
"""
from .model import (  # noqa: F401
    DecodeState, OracleModel, apply_rope, argmax_lowest, attention_one_query,
    causal_attention, rms_norm, rope_cos_sin, rope_inv_freq, silu, top2_margin,
)

"""Shared helpers of the parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, and compare by the stated bar:

  * logits, every compared step: max |gpu - oracle| <= 1e-2 * max |oracle|;
  * greedy ids: identical wherever the oracle's top-1 minus top-2 logit
    margin exceeds 2e-2 (absolute logit units).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

import synth
from oracle import OracleModel, top2_margin

LOGIT_RTOL = 1e-2      # of max |oracle logit| at that step
MARGIN = 2e-2          # ids must agree where the oracle's top-2 margin exceeds this


@dataclasses.dataclass
class StepReport:
    compared: int
    worst_rel: float
    id_checked: int
    first_divergence: Optional[int]


def compare_steps(gpu_logits: np.ndarray, gpu_ids: np.ndarray, ref_logits: np.ndarray) -> StepReport:
    """Teacher-forced comparison: row i of both logit arrays comes from the
    same fed prefix; gpu_ids[i] is the GPU's pick from its row i."""
    n = ref_logits.shape[0]
    assert gpu_logits.shape == ref_logits.shape, (gpu_logits.shape, ref_logits.shape)
    worst = 0.0
    checked = 0
    for i in range(n):
        ref = ref_logits[i].astype(np.float64)
        got = gpu_logits[i].astype(np.float64)
        assert np.all(np.isfinite(got)), f"non-finite GPU logits at step {i}"
        scale = np.max(np.abs(ref))
        err = np.max(np.abs(got - ref))
        rel = err / scale
        worst = max(worst, rel)
        assert err <= LOGIT_RTOL * scale, (
            f"step {i}: max|dlogit| {err:.3e} > {LOGIT_RTOL} * {scale:.3e}")
        if top2_margin(ref) > MARGIN:
            checked += 1
            assert int(gpu_ids[i]) == int(np.argmax(ref)), (
                f"step {i}: gpu id {gpu_ids[i]} != oracle argmax {np.argmax(ref)} "
                f"(margin {top2_margin(ref):.3e})")
        # the pick must be the argmax of the GPU's own logits (bit-exact decision)
        assert int(gpu_ids[i]) == int(np.argmax(gpu_logits[i])), f"step {i}: pick != own argmax"
    return StepReport(n, worst, checked, None)


def compare_free_running(gpu_ids: List[int], gpu_logits: np.ndarray, or_ids: List[int],
                         or_logits: np.ndarray) -> StepReport:
    """Free-running greedy: compare while the fed prefixes agree; a difference
    is allowed only at a step where the oracle's margin is <= MARGIN, and the
    comparison ends there (the sequences legitimately diverge)."""
    n = min(len(gpu_ids), len(or_ids))
    worst = 0.0
    checked = 0
    for i in range(n):
        ref = or_logits[i].astype(np.float64)
        got = gpu_logits[i].astype(np.float64)
        scale = np.max(np.abs(ref))
        err = np.max(np.abs(got - ref))
        worst = max(worst, err / scale)
        assert err <= LOGIT_RTOL * scale, (
            f"step {i}: max|dlogit| {err:.3e} > {LOGIT_RTOL} * {scale:.3e}")
        m = top2_margin(ref)
        if gpu_ids[i] != or_ids[i]:
            assert m <= MARGIN, f"step {i}: ids differ ({gpu_ids[i]} vs {or_ids[i]}) at margin {m:.3e}"
            return StepReport(i + 1, worst, checked, i)
        if m > MARGIN:
            checked += 1
    return StepReport(n, worst, checked, None)


def device_model(model: synth.SynthModel):
    from persistent_sm_decode_monokernel_b200 import upload_weights
    return upload_weights(model.tensors)

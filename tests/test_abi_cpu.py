"""The C ABI on the CPU: libkie.so builds, loads, exports every symbol the
header declares, and its host-only calls (shape checks, KV sizing, the CTA
work partition) behave.  No CUDA compute call is made here."""
import ctypes
import os
import re

import pytest

import synth
from persistent_sm_decode_monokernel_b200 import _kie, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _kie.load_library()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "kie.h")).read()
    return sorted(set(re.findall(r"KIE_API[^;(]*?\b(kie_\w+)\s*\(", text)))


def test_header_symbols_exported(lib):
    names = _declared_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
        assert n in _kie.SIGNATURES, f"binding lacks {n}"


def _desc(shape, max_seq=64, eos=-1):
    return _kie.make_desc(shape.n_layers, shape.d_model, shape.n_heads, shape.n_kv_heads,
                          shape.head_dim, shape.ffn_dim, shape.vocab, shape.rope_base,
                          shape.rms_eps, max_seq, eos)


def test_check_desc_accepts_all_workloads(lib):
    for w in synth.WORKLOADS.values():
        assert _kie.kie_check_desc(_desc(w.shape, w.max_seq)) == _kie.KIE_OK


@pytest.mark.parametrize("change,status", [
    (dict(head_dim=96), _kie.KIE_ERR_UNSUPPORTED),
    (dict(n_heads=6, n_kv_heads=4), _kie.KIE_ERR_UNSUPPORTED),
    (dict(n_heads=36, n_kv_heads=4), _kie.KIE_ERR_UNSUPPORTED),
    (dict(d_model=320), _kie.KIE_ERR_UNSUPPORTED),
    (dict(ffn_dim=1000), _kie.KIE_ERR_UNSUPPORTED),
    (dict(n_layers=0), _kie.KIE_ERR_INVALID_ARG),
    (dict(vocab=0), _kie.KIE_ERR_INVALID_ARG),
])
def test_check_desc_rejects(lib, change, status):
    base = dict(n_layers=2, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64, ffn_dim=768,
                vocab=2048)
    base.update(change)
    assert _kie.kie_check_desc(_desc(synth.ModelShape(**base))) == status


def test_check_desc_rejects_bad_eos_and_capacity(lib):
    s = synth.WORKLOADS["tiny-l2-d256"].shape
    assert _kie.kie_check_desc(_desc(s, 48, eos=2048)) == _kie.KIE_ERR_INVALID_ARG
    assert _kie.kie_check_desc(_desc(s, 48, eos=-2)) == _kie.KIE_ERR_INVALID_ARG
    assert _kie.kie_check_desc(_desc(s, 0)) == _kie.KIE_ERR_INVALID_ARG
    assert _kie.kie_check_desc(None) == _kie.KIE_ERR_INVALID_ARG


def test_kv_cache_bytes(lib):
    for w in synth.WORKLOADS.values():
        s = w.shape
        want = 2 * s.n_layers * s.n_kv_heads * w.max_seq * (s.head_dim + 8) * 2   # padded rows
        assert _kie.kie_kv_cache_bytes(_desc(s, w.max_seq)) == want
    bad = _desc(synth.WORKLOADS["tiny-l2-d256"].shape, 0)
    assert _kie.kie_kv_cache_bytes(bad) == 0


def _units(s, st):
    hd = s.head_dim
    return [s.n_heads * hd // 2 + s.n_kv_heads * hd // 2 + s.n_kv_heads * hd, s.d_model,
            s.ffn_dim, s.d_model, s.vocab][st]


def _rows(s, st, ub, ue):
    if st == 0:
        npairs = (s.n_heads + s.n_kv_heads) * s.head_dim // 2
        npr = max(0, min(ue, npairs) - ub)
        return 2 * npr + (ue - ub - npr)
    if st == 2:
        return 2 * (ue - ub)
    return ue - ub


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_partition_covers_and_balances(lib, name):
    s = synth.WORKLOADS[name].shape
    d = _desc(s)
    grid = 148
    for st in range(5):
        rng = [_kie.kie_plan_units(d, grid, st, c) for c in range(grid)]
        srt = sorted(rng)
        assert srt[0][0] == 0 and srt[-1][1] == _units(s, st)
        assert all(a[1] == b[0] for a, b in zip(srt, srt[1:])), "ranges must tile the units"
        rows = [_rows(s, st, a, b) for a, b in rng]
        assert sum(rows) == {0: (s.n_heads + 2 * s.n_kv_heads) * s.head_dim, 1: s.d_model,
                             2: 2 * s.ffn_dim, 3: s.d_model, 4: s.vocab}[st]
        unit_rows = 2 if st in (0, 2) else 1
        assert max(rows) - min(rows) <= 2 * unit_rows - 1 + (st == 0), (st, max(rows), min(rows))
    # O and down share one partition (each CTA keeps its residual rows)
    for c in range(grid):
        assert _kie.kie_plan_units(d, grid, 1, c) == _kie.kie_plan_units(d, grid, 3, c)
    # elsewhere the CTAs that carry an extra unit differ between stages
    big = []
    for st in (1, 4):
        rows = [_rows(s, st, *_kie.kie_plan_units(d, grid, st, c)) for c in range(grid)]
        big.append({c for c in range(grid) if rows[c] == max(rows)})
    assert big[0] != big[1] or len(big[0]) == grid


def test_plan_units_rejects_bad_args(lib):
    d = _desc(synth.WORKLOADS["tiny-l2-d256"].shape)
    b, e = ctypes.c_int32(), ctypes.c_int32()
    L = lib
    assert L.kie_plan_units(ctypes.byref(d), 0, 0, 0, ctypes.byref(b), ctypes.byref(e)) == 1
    assert L.kie_plan_units(ctypes.byref(d), 4, 5, 0, ctypes.byref(b), ctypes.byref(e)) == 1
    assert L.kie_plan_units(ctypes.byref(d), 4, 0, 4, ctypes.byref(b), ctypes.byref(e)) == 1


def test_status_strings(lib):
    for s in range(10):
        assert lib.kie_status_str(s) != b"unknown status"
    assert lib.kie_status_str(99) == b"unknown status"


def test_selection_setters_reject_null_context(lib):
    assert lib.kie_set_sampling(None, 1.0, 5) == _kie.KIE_ERR_INVALID_ARG
    assert lib.kie_set_sampling_filter(None, 5, 0.9) == _kie.KIE_ERR_INVALID_ARG
    ids = (ctypes.c_int32 * 2)(1, 2)
    assert lib.kie_set_eos_ids(None, ids, 2) == _kie.KIE_ERR_INVALID_ARG
    assert _kie.KIE_MAX_EOS_IDS == int(re.search(
        r"#define KIE_MAX_EOS_IDS (\d+)", open(os.path.join(ROOT, "include", "kie.h")).read()).group(1))


C_CLIENT = r"""
#include <stdio.h>
#include "kie.h"

int main(void) {
  kie_model_desc d;
  int32_t b = -1, e = -1;
  d.n_layers = 2; d.d_model = 256; d.n_heads = 4; d.n_kv_heads = 4; d.head_dim = 64;
  d.ffn_dim = 768; d.vocab = 2048; d.rope_base = 10000.0f; d.rms_eps = 1e-5f;
  d.max_seq = 48; d.eos_id = -1;
  printf("check %d\n", (int)kie_check_desc(&d));
  printf("kv %lu\n", (unsigned long)kie_kv_cache_bytes(&d));
  printf("plan %d", (int)kie_plan_units(&d, 148, 4, 3, &b, &e));
  printf(" %d %d\n", (int)b, (int)e);
  printf("sampling %d\n", (int)kie_set_sampling(NULL, 1.0f, 7u));
  printf("eos %d %d\n", (int)kie_set_eos_ids(NULL, NULL, 0), KIE_MAX_EOS_IDS);
  printf("str %s\n", kie_status_str(KIE_ERR_CAPACITY));
  return 0;
}
"""


def test_header_is_plain_c_and_links(lib, tmp_path):
    """A C99 program compiles against include/kie.h with warnings as errors,
    links libkie.so and gets the same answers from the host-only calls."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(_kie.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-l:libkie.so", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    s = synth.WORKLOADS["tiny-l2-d256"].shape
    d = _desc(s, 48)
    b, e = _kie.kie_plan_units(d, 148, 4, 3)
    assert out[0] == "check 0"
    assert out[1] == f"kv {2 * 2 * 4 * 48 * (64 + 8) * 2}"
    assert out[2] == f"plan 0 {b} {e}"
    assert out[3] == f"sampling {_kie.KIE_ERR_INVALID_ARG}"
    assert out[4] == f"eos {_kie.KIE_ERR_INVALID_ARG} {_kie.KIE_MAX_EOS_IDS}"
    assert out[5] == "str " + lib.kie_status_str(_kie.KIE_ERR_CAPACITY).decode()

#!/usr/bin/env python
"""Batch-1 decode benchmark of the persistent decode kernel on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--temperature T --seed S] [--impl reference] [--no-cpu-baseline]

A step is one request's decode: the session is rewound to the end of the
prompt (P positions of KV already in HBM) and kie_decode runs S steps
(greedy, or temperature sampling with --temperature) in ONE launch of the
persistent kernel.  W untimed steps, then K timed
steps bracketed by a barrier and a device synchronize, timed with CUDA
events on the launching stream.  `value` is decode tokens/s per request:
N * K * S / (max over ranks of the timed region).  With N > 1 every rank
runs an independent replica (the path does not shard; there is no
collective on the data path).

`--impl reference` times the CPU oracle instead (rank 0 only), on a bounded
sample of the same workload, and prints the same JSON line with
"impl": "reference".

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

DEFAULT_WORKLOAD = "l28-d2560"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
METRIC = "batch-1 decode tokens/s per request"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = ["kie_kernel.cu", "kie_device.cuh", "kie_params.h", "kie_units.h"]


def kernel_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "persistent_sm_decode_monokernel_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(w: synth.Workload, n_steps: int):
    """DRAM bytes per launch from the committed ncu summary of this workload
    (bytes per decode step x steps), or None when the summary is missing or
    was taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", f"monokernel_{w.name}_traffic.md")
    try:
        text = open(path).read()
    except OSError:
        return None, "no profile summary"
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip().split()[0] if v.strip() else ""
    if vals.get("kernel_source_sha256") != kernel_sha():
        return None, "kernel changed since the ncu capture"
    try:
        per_step = float(vals["dram_bytes_per_step"])
    except (KeyError, ValueError):
        return None, "summary lacks dram_bytes_per_step"
    return per_step * n_steps, path


def weight_bytes_per_token(s: synth.ModelShape, weights: str = "fp16") -> float:
    """Bytes of the weights one decode step reads: every matrix (fp16, or
    one byte per FP8 E4M3 code plus a 4-byte scale per row), the fp16 norm
    gains and one fp16 embedding row."""
    if weights == "fp16":
        return float(s.matrix_bytes_per_token())
    d, L = s.d_model, s.n_layers
    rows = L * (s.q_dim + 2 * s.kv_dim + d + 2 * s.ffn_dim + d) + s.vocab
    elems = L * (d * s.q_dim + 2 * d * s.kv_dim + s.q_dim * d + 3 * d * s.ffn_dim) + s.vocab * d
    return float(elems + 4 * rows + 2 * (2 * L * d + d) + 2 * d)


def decode_bytes(w: synth.Workload, pos0: int, n_steps: int, weights: str = "fp16") -> float:
    """Algorithmic HBM bytes of n_steps decode steps starting at position
    pos0: every weight matrix, the norm gains and one embedding row per
    step, plus K/V reads of positions 0..pos and the K/V write at pos."""
    s = w.shape
    per_pos = s.kv_bytes_per_position()
    wb = weight_bytes_per_token(s, weights)
    total = 0.0
    for i in range(n_steps):
        pos = pos0 + i
        total += wb + per_pos * (pos + 1) + per_pos
    return total


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(parts)
            except ValueError:
                pass
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        # samples under load: the upper half by power draw
        loaded = sm
        if power and len(power) == len(sm):
            thr = statistics.median(power)
            loaded = [s for s, p in zip(sm, power) if p >= thr] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4)
                          if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------ distribution

def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world <= 1:
        return None, 0, 1
    import torch.distributed as dist
    from datetime import timedelta
    backend = os.environ.get("KIE_BENCH_BACKEND", "nccl")
    dist.init_process_group(backend=backend, timeout=timedelta(seconds=300))
    return dist, dist.get_rank(), dist.get_world_size()


def reduce_max_sum(dist, elapsed_s: float, tokens: float, device=None):
    """(max over ranks of elapsed, sum over ranks of tokens)."""
    if dist is None:
        return elapsed_s, tokens
    import torch
    t = torch.tensor([elapsed_s], dtype=torch.float64, device=device)
    n = torch.tensor([tokens], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), float(n.item())


# ------------------------------------------------------------- CPU oracle

def cpu_oracle_rate(w: synth.Workload, model, budget_s: float = 15.0, max_steps: int = 256,
                    warmup: int = 1, single_budget_s: float = 8.0):
    """Times the oracle's incremental decode (fp32, numpy/BLAS) after a
    batched prefill of the prompt: on all host cores (BLAS threads), then on
    one thread (BLAS limited to 1) for a shorter sample continuing from the
    same state.  Returns (tok/s all cores, info)."""
    from oracle import OracleModel, argmax_lowest
    from threadpoolctl import threadpool_info, threadpool_limits
    om = OracleModel(model, dtype=np.float32)
    prompt = synth.make_prompt(w.shape.vocab, w.prompt_len, seed=w.seed)
    t0 = time.perf_counter()
    st, lg = om.prefill_batched(prompt)
    t_prefill = time.perf_counter() - t0
    tok = argmax_lowest(lg)
    for _ in range(warmup):
        tok = argmax_lowest(om.decode_step(st, tok))

    def timed(budget):
        nonlocal tok
        n = 0
        t0 = time.perf_counter()
        while n < max_steps and (time.perf_counter() - t0) < budget:
            tok = argmax_lowest(om.decode_step(st, tok))
            n += 1
        return n, time.perf_counter() - t0

    first = st.pos
    n, el = timed(budget_s)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    info = {"steps": n, "seconds": el, "prefill_s": t_prefill, "threads": threads,
            "first_pos": first, "nproc": os.cpu_count()}
    if single_budget_s > 0:
        first1 = st.pos
        with threadpool_limits(limits=1):
            n1, el1 = timed(single_budget_s)
        info["single_thread"] = {"value": n1 / el1, "unit": "tok/s", "cores": 1,
                                 "sample": f"{n1} fp32 oracle decode steps at positions "
                                           f"{first1}+ on one thread ({el1:.1f} s timed)"}
    return n / el, info


# ------------------------------------------------------------------ arms

def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    model = synth.make_model(w.shape, seed=w.seed)
    from oracle import OracleModel, argmax_lowest
    from oracle import sampling
    from threadpoolctl import threadpool_info
    om = OracleModel(model, dtype=np.float32)
    prompt = synth.make_prompt(w.shape.vocab, w.prompt_len, seed=w.seed)
    st, lg = om.prefill_batched(prompt)

    def pick(logits, pos):
        if args.temperature > 0:
            return sampling.sample_id(logits, args.temperature, args.seed, pos)
        return argmax_lowest(logits)

    tok = pick(lg, w.prompt_len - 1)
    per_step = args.ref_tokens_per_step

    def step():
        nonlocal tok
        pos = st.pos
        tok = pick(om.decode_step(st, tok), pos)

    for _ in range(args.warmup):
        for _ in range(per_step):
            step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for _ in range(per_step):
            step()
    el = time.perf_counter() - t0
    value = args.steps * per_step / el
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    sample = (f"{per_step} oracle decode steps per bench step (fp32 numpy, cached fp32 weights) "
              f"at positions {w.prompt_len}+ after a batched prefill of the {w.prompt_len}-id "
              f"prompt; {args.steps} timed bench steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * el / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": run_config(w, args),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": threads, "kind": "oracle",
                         "host_nproc": os.cpu_count(), "sample": sample},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_config(w: synth.Workload, args):
    """The workload plus the token-selection rule and weight format of this run."""
    sel = "greedy" if args.temperature <= 0 else {
        "sampling": "temperature (Gumbel-max, Philox4x64-10)",
        "temperature": args.temperature, "seed": args.seed,
        "top_k": args.top_k, "top_p": args.top_p}
    cfg = dict(workload_config(w), token_selection=sel)
    if getattr(args, "weights", "fp16") == "fp8":
        cfg["weights"] = ("fp16 N(0,0.02), seed 0, streamed as FP8 E4M3 with one fp32 "
                          "scale per row (quantised by the library)")
        cfg["weight_bytes_per_token"] = weight_bytes_per_token(w.shape, "fp8")
    return cfg


def workload_config(w: synth.Workload):
    s = w.shape
    return {"workload": w.name, "layers": s.n_layers, "d_model": s.d_model,
            "heads": s.n_heads, "kv_heads": s.n_kv_heads, "head_dim": s.head_dim,
            "ffn": s.ffn_dim, "vocab": s.vocab, "params": s.n_params(),
            "prompt_len": w.prompt_len, "decode_steps_per_launch": w.decode_steps,
            "batch": 1, "weights": "fp16 N(0,0.02), seed 0", "kv_cache": "fp16",
            "parallelism": "replicas",
            "l2": "inputs larger than L2 (weights streamed per token exceed the 126 MB L2)"}


def run_gpu(args, w, dist, rank, world):
    import torch
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    from persistent_sm_decode_monokernel_b200 import Session, build, upload_weights
    if rank == 0 or not os.path.exists(os.path.join(ROOT, "persistent_sm_decode_monokernel_b200",
                                                      "libkie.so")):
        build.build()
    if dist is not None:
        dist.barrier()
    model = synth.make_model(w.shape, seed=w.seed)
    dev = upload_weights(model.tensors)
    prompt = synth.make_prompt(w.shape.vocab, w.prompt_len, seed=w.seed)
    stream = torch.cuda.current_stream()
    # the session keeps the caller's fp16 matrices: the batched prefill
    # (tensor-core GEMMs over the prompt) reads them
    sess = Session(w.shape, dev, max_seq=w.max_seq, stream=stream, weight_format=args.weights)
    sess.set_sampling(args.temperature, args.seed, top_k=args.top_k, top_p=args.top_p)
    # the prompt's prefill, timed on its own (the second run: the first
    # allocates the prefill scratch); decode is what the metric measures
    sess.prefill(prompt)
    sess.prefill(prompt)
    pst = sess.stats()
    P, S = w.prompt_len, w.decode_steps
    prefill_info = {"ms": pst["last_prefill_ms"], "positions": P,
                    "path": ("batched: tcgen05 GEMMs over positions 0..P-2, the last position "
                             "as one decode step") if pst["last_prefill_batched"] else
                            "one decode step per position",
                    "tokens_per_s": P / (pst["last_prefill_ms"] * 1e-3)}
    out = np.empty(S, dtype=np.int32)

    def one_step():
        sess.rewind(P)
        ids = sess.decode(S, out)
        assert len(ids) == S
        return sess.stats()["last_device_ms"]

    for _ in range(args.warmup):
        one_step()
    ref_ids = out.copy()

    clocks = ClockSampler(local)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    launch_ms = []
    ev0.record(stream)
    for _ in range(args.steps):
        launch_ms.append(one_step())
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if dist is not None:
        dist.barrier()
    elapsed = ev0.elapsed_time(ev1) / 1000.0
    deterministic = bool(np.array_equal(out, ref_ids))
    t_max, tokens = reduce_max_sum(dist, elapsed, float(args.steps * S),
                                   device=torch.device("cuda", local))
    value = tokens / t_max

    # end to end through the public call with host buffers, host clock
    e2e_times = []
    for _ in range(max(1, min(args.steps, 3))):
        sess.rewind(P)
        t0 = time.perf_counter()
        sess.decode(S, out)
        e2e_times.append(time.perf_counter() - t0)
    e2e_local = sum(e2e_times)
    e2e_max, e2e_tok = reduce_max_sum(dist, e2e_local, float(len(e2e_times) * S),
                                      device=torch.device("cuda", local))

    st = sess.stats()
    loop = st["loop_cycles"] or 1.0
    sync_frac = st["sync_wait_cycles"] / loop
    stream_frac = st["stream_wait_cycles"] / loop
    sess.close()

    if rank != 0:
        return 0
    peak, peak_kind = _peaks()
    avg_launch_s = (sum(launch_ms) / len(launch_ms)) / 1000.0
    bytes_launch = decode_bytes(w, P, S, args.weights)
    achieved = bytes_launch / avg_launch_s / 1e9
    traffic, traffic_src = profiled_traffic(w, S)
    if args.traffic is not None:
        traffic, traffic_src = args.traffic, "command line"
    line = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * t_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": ("f16 weights+KV, f16 GEMV inputs, f32 accumulate" if args.weights == "fp16"
                  else "fp8 E4M3 weights (fp32 row scales), f16 KV, f16 GEMV inputs, "
                       "f32 accumulate"),
        "data": "synthetic",
        "config": run_config(w, args),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind,
                     "frac_vs_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "traffic": traffic, "traffic_source": traffic_src,
                     "algorithmic_bytes_per_launch": bytes_launch,
                     "avg_launch_ms": avg_launch_s * 1000.0},
        "e2e": {"value": e2e_tok / e2e_max, "unit": "tok/s",
                "h2d_bytes_per_step": 4, "d2h_bytes_per_step": 4 * S + 32,
                "how": "host clock around kie_decode (host id buffer): launch, device run, "
                       "D2H of ids and status"},
        "gpu_launches": args.steps,
        "clocks": clk,
        "sync_wait_frac": sync_frac, "stream_wait_frac": stream_frac,
        "per_token_us": 1e6 * avg_launch_s / S,
        "deterministic_ids": deterministic,
        "prefill": prefill_info,
    }
    if not args.no_cpu_baseline:
        rate, info = cpu_oracle_rate(w, model)
        line["cpu_baseline"] = {
            "value": rate, "unit": "tok/s", "cores": info["threads"], "kind": "oracle",
            "host_nproc": info["nproc"],
            "sample": f"{info['steps']} fp32 oracle decode steps at positions "
                      f"{info['first_pos']}+ after a batched prefill of the prompt, "
                      f"BLAS on {info['threads']} threads of {info['nproc']} host cores "
                      f"({info['seconds']:.1f} s timed)"}
        if "single_thread" in info:
            line["cpu_baseline"]["single_thread"] = info["single_thread"]
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(synth.WORKLOADS) + sorted(synth.PROFILE_WORKLOADS))
    ap.add_argument("--decode-steps", type=int, default=None,
                    help="decode steps per launch (default: the workload's); for profiler runs")
    ap.add_argument("--weights", default="fp16", choices=["fp16", "fp8"],
                    help="weight stream format: fp16 (default) or FP8 E4M3 with row scales")
    ap.add_argument("--top-k", type=int, default=0, help="sampling: top-k bound (0 = off)")
    ap.add_argument("--top-p", type=float, default=1.0, help="sampling: nucleus (1 = off)")
    ap.add_argument("--temperature", type=float, default=0.0,
                    help="0 = greedy (default); > 0 = in-kernel temperature sampling")
    ap.add_argument("--seed", type=int, default=0, help="sampling seed")
    ap.add_argument("--impl", default="kie", choices=["kie", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-tokens-per-step", type=int, default=4)
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch from an ncu capture of the same kernel")
    args = ap.parse_args(argv)
    w = synth.workload(args.workload)
    if args.decode_steps is not None:
        import dataclasses
        w = dataclasses.replace(w, decode_steps=args.decode_steps)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
        return run_reference(args, w, rank, world)
    dist, rank, world = init_dist()
    try:
        return run_gpu(args, w, dist, rank, world)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())

"""The benchmark's host-side logic on the CPU: the byte accounting of the
roofline, and the multi-rank aggregation (max of the timed region, sum of
tokens over ranks) run as two gloo ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
import synth


def test_decode_bytes_matches_mean_formula():
    for name in ("l28-d2560", "l28-d2560-ctx8k", "l32-d4096"):
        w = synth.WORKLOADS[name]
        total = bench.decode_bytes(w, w.prompt_len, w.decode_steps)
        assert abs(total / w.decode_steps - w.bytes_per_token_mean()) / total < 1e-9


def test_decode_bytes_counts_weights_and_kv():
    w = synth.WORKLOADS["l28-d2560"]
    s = w.shape
    one = bench.decode_bytes(w, 0, 1)
    # position 0 reads one position of K/V and writes one
    assert one == s.matrix_bytes_per_token() + 2 * s.kv_bytes_per_position()


def _free_port():
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    t, n = bench.reduce_max_sum(dist, elapsed_s=1.0 + rank, tokens=100.0 * (rank + 1))
    out[rank] = (t, n)
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_max_sum_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == out[1] == (2.0, 300.0)


def test_single_process_is_identity():
    assert bench.reduce_max_sum(None, 3.5, 7.0) == (3.5, 7.0)


def test_profiled_traffic_rejects_other_kernel(tmp_path, monkeypatch):
    w = synth.WORKLOADS["l28-d2560"]
    traffic, why = bench.profiled_traffic(w, 1024)
    assert traffic is None or traffic > 0


def test_reference_arm_under_torchrun_prints_one_line_on_rank0():
    """`bench.py --impl reference` launched like the GPU arm (two ranks):
    rank 0 times the oracle and prints the contract's JSON line, the other
    rank exits 0 without work."""
    import json
    import subprocess
    import sys
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(bench.ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny-l2-d256",
           "--gpus", "2", "--steps", "2", "--warmup", "1", "--temperature", "0.9", "--seed", "5"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=bench.ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tok/s" and d["value"] > 0
    assert d["n_gpus"] == 2 and d["steps"] == 2 and d["warmup"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tok/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["token_selection"]["temperature"] == 0.9

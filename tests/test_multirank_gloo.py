"""Host logic of the multi-GPU replicas on CPU: two gloo ranks, the same weights on each,
different tokens per rank, the step time reduced as the max over ranks and the whole-job
throughput counted over all ranks' tokens. (The layer needs no collective: tokens are
independent, so ranks are data-parallel replicas.)"""
import hashlib
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _digest(t):
    return hashlib.sha256(t.contiguous().view(torch.int16).numpy().tobytes()).hexdigest()


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    from deterministic_invariant_routing_b200 import synthetic
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, loc = bench.dist_env()
        s = synthetic.shape("tiny", T=32)
        weights, x = bench.replica_inputs(s, r, "cpu")
        step_ms = 1.0 + r  # rank 1 is the slow one
        ms = bench.reduce_max(step_ms, "cpu", w)
        info = {"rank": r, "world": w, "local": loc, "ms_max": ms,
                "w13": _digest(weights["w13"]), "x": _digest(x),
                "value": bench.job_tokens_per_s(s.T, w, ms)}
        gathered = [None] * w
        dist.all_gather_object(gathered, info)
        if r == 0:
            out.put(gathered)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_are_replicas_with_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = q.get(timeout=180)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    a, b = sorted(res, key=lambda d: d["rank"])
    assert (a["world"], b["world"]) == (2, 2) and (a["local"], b["local"]) == (0, 1)
    assert a["ms_max"] == b["ms_max"] == 2.0
    assert a["w13"] == b["w13"]          # the same layer on every rank
    assert a["x"] != b["x"]              # each rank its own tokens
    assert a["value"] == pytest.approx(32 * 2 / 2e-3)


def test_single_process_defaults():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, "cpu", 1) == 3.5
    assert bench.job_tokens_per_s(16384, 1, 1.6) == pytest.approx(16384 / 1.6e-3)


def test_reference_arm_line_on_cpu():
    """`bench.py --impl reference` times the oracle on the host and prints one JSON line with
    the reference arm's keys (no GPU needed)."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--T", "64", "--steps", "1", "--warmup", "1"], cwd=root,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "tiny_T64"

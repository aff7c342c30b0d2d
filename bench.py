#!/usr/bin/env python
"""MoE-layer throughput on B200: tokens/s of the batch-invariant top-k MoE FFN forward
(bf16, fp32 accumulate) and its fraction of the tensor/HBM roofline.

One step = one moe_forward over a batch of synthetic tokens already resident in HBM:
router logits -> routing -> dispatch -> grouped gate_up/SwiGLU -> grouped down ->
(shared expert) -> fixed-order combine. Default workload: the Qwen3-30B-A3B-shaped layer
(hidden 2048, 128 experts x 768, top-8 softmax, renormalised) at T = 16384 tokens.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 launch one process per GPU with torch.distributed.run; every rank runs an
independent replica of the layer on its own tokens (the layer has no cross-token
exchange), the time is the max over ranks, and value = all ranks' tokens / that time.
`--impl reference` times the plain CPU oracle (the correctness reference, run as it
stands on the host cores) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CPU_SAMPLE_SECONDS = 15.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="qwen3_30b_a3b")
    p.add_argument("--T", type=int, default=16384)
    p.add_argument("--e2e-steps", type=int, default=0, help="0: same as --steps")
    p.add_argument("--e2e-chunk", type=int, default=6144,
                   help="tokens per chunk of the host-memory call (copies overlap compute)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extras", action="store_true",
                   help="skip timing the order-invariant combine, the router statistics and "
                        "the backward")
    p.add_argument("--extras-reps", type=int, default=20,
                   help="timed repetitions of each extra call")
    p.add_argument("--split-steps", type=int, default=200,
                   help="steps of the separate pass that records the per-stage events")
    p.add_argument("--sweep", action="store_true",
                   help="instead of the bench line: tokens/s of the layer forward at each batch "
                        "size of the invariance sweep (one JSON object)")
    p.add_argument("--oracle-sweep", action="store_true",
                   help="instead of the bench line: the oracle's tokens/s on the host cores for "
                        "each workload (one JSON object)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_sha(rels):
    """Hash of the kernel's source files (a list of repo-relative paths)."""
    h = hashlib.sha256()
    for rel in rels:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, rows, layer, workload=None):
    """DRAM bytes (read + write) per launch of a kernel, from a committed ncu summary
    (profiles/ncu_traffic.json): the single-launch capture of this workload when there is
    one, else the straight line through the captures at two smaller sizes of the same layer
    (fixed bytes of the weights plus bytes per routed row) at `rows`. None for a layer the
    record does not cover, or when the kernel's sources changed since the counters were
    taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel_key]
        if rec["source_sha"] != source_sha(rec["sources"]):
            return None
        if rec.get("layer") != layer:
            return None
        cap = rec.get("captures", {}).get(workload)
        if cap is not None and cap["routed_rows"] == rows:
            return cap["bytes"]
        return round(rec["fixed_bytes"] + rec["bytes_per_row"] * rows)
    except Exception:
        return None


class ClockSampler:
    """SM clock, power and throttle reasons sampled while the timed region runs.

    NVML is read from a thread every few milliseconds (reading only; no setting is
    touched), so that even a timed region of a few tens of milliseconds gets several
    samples; nvidia-smi at its 100 ms floor is the fallback when NVML is missing."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id, period_s=0.002):
        self.gpu_id = gpu_id
        self.period_s = period_s
        self.proc = None
        self.thread = None
        self.samples = []      # (sm MHz, max MHz, set of reason names)
        self.source = None

    def _nvml_loop(self, nv, h):
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self.stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, mx, {n for n, b in bits.items() if r & b}))
            except Exception:
                pass
            self.stop.wait(self.period_s)

    def __enter__(self):
        import threading
        self.stop = threading.Event()
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByUUID(self.gpu_id) if self.gpu_id.startswith("GPU-") \
                else nv.nvmlDeviceGetHandleByIndex(int(self.gpu_id))
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.thread.start()
            # the first reading before the timed region starts, so that a region of a few
            # milliseconds is still sampled
            t0 = time.perf_counter()
            while not self.samples and time.perf_counter() - t0 < 0.5:
                time.sleep(0.0005)
            self.source = f"NVML every {self.period_s * 1e3:.0f} ms"
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.gpu_id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi every 100 ms"
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            for l in out.splitlines():
                f = [x.strip() for x in l.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm, mx = float(f[1]), float(f[2])
                except ValueError:
                    continue
                self.samples.append((sm, mx, {n for n, v in zip(self.NAMES, f[5:9])
                                              if v.lower() == "active"}))

    def summary(self):
        # samples from the start of the timed region on (plus the one reading just before it)
        sm = [a for a, _, _ in self.samples]
        mx = max((b for _, b, _ in self.samples), default=0.0)
        reasons = set()
        for _, _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": mx or None, "reasons": sorted(reasons), "samples": len(sm),
                "source": self.source}


def dist_env():
    """(rank, world size, local rank) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max(v, dev, world):
    """The max of a per-rank number over all ranks (the slowest rank's time)."""
    if world == 1:
        return float(v)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_inputs(s, rank, device):
    """Each rank is a replica: the same weights everywhere, its own tokens."""
    from deterministic_invariant_routing_b200 import synthetic
    weights = synthetic.make_weights(s, device=device)
    x = synthetic.make_tokens(s, s.T, seed=s.seed + 1000 * rank, device=device)
    return weights, x


def job_tokens_per_s(T_per_rank, world, ms_max):
    """Whole-job throughput: every rank's tokens over the slowest rank's step time."""
    return T_per_rank * world / (ms_max * 1e-3)


def layer_work(s, n_touched):
    """Algorithmic FLOPs and bytes of one layer forward (intermediates excluded)."""
    T, H, E, K, I, Is = s.T, s.H, s.E, s.K, s.I, s.I_shared
    flops = T * K * (4 * H * I + 2 * I * H) + T * 6 * H * Is + 2 * T * H * E
    byts = (n_touched * 3 * H * I * 2 + 3 * H * Is * 2 + 2 * T * H * 2 + E * H * 2
            + T * K * 8)
    return flops, byts


def _calibrate(s, d_cpu):
    """Seconds per token of the oracle's layer forward with every host core busy."""
    import numpy as np

    import oracle
    n = max(oracle.num_threads(), 2)
    sel = np.arange(min(n, s.T), dtype=np.int32)
    t0 = time.perf_counter()
    oracle.layer_forward(s, d_cpu, sel)
    return max((time.perf_counter() - t0) / sel.size, 1e-6)


def cpu_baseline(s, d_cpu, seconds=CPU_SAMPLE_SECONDS, per_tok=None, seed=0):
    """The oracle's whole-layer forward on a bounded token sample, tokens/s."""
    import numpy as np

    import oracle
    rng = np.random.default_rng(seed)
    if per_tok is None:
        per_tok = _calibrate(s, d_cpu)
    n = int(min(max(seconds / per_tok, 1), s.T))
    sel = np.sort(rng.choice(s.T, n, replace=False)).astype(np.int32)
    t0 = time.perf_counter()
    oracle.layer_forward(s, d_cpu, sel)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} of the {s.T} tokens of the same layer (full layer per token: FP64 "
                      f"router, FP32-contract routing, FP64 experts), {dt:.2f} s"}


def run_reference(a):
    """The correctness reference (the CPU oracle, as it stands) on the host cores; each
    step is a bounded token sample, the whole run about 90 s."""
    from deterministic_invariant_routing_b200 import synthetic
    rank, _, _ = dist_env()
    if rank != 0:
        return
    s, d = synthetic.make_layer(a.workload, T=a.T, device="cpu")
    per_tok = _calibrate(s, d)
    secs = max(90.0 / (a.warmup + a.steps), per_tok)
    per_step, step_ms = [], []
    for i in range(a.warmup + a.steps):
        t0 = time.perf_counter()
        r = cpu_baseline(s, d, seconds=secs, per_tok=per_tok, seed=i)
        if i >= a.warmup:
            per_step.append(r)
            step_ms.append(1e3 * (time.perf_counter() - t0))
    value = statistics.median(r["value"] for r in per_step)
    cb = dict(per_step[-1], value=value)
    cb["sample"] = f"per step: {per_step[-1]['sample']}"
    # each timed step is a token sample of the workload, so ms_per_step is that sample's
    # measured time; the full batch's time is extrapolated from the rate and labelled so
    line = {"impl": "reference", "metric": "MoE-layer tokens/s (bf16, batch-invariant)",
            "value": value, "unit": "tokens/s", "n_gpus": a.gpus, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": statistics.median(step_ms),
            "ms_per_step_kind": "measured: one step = one bounded token sample",
            "ms_per_full_batch_extrapolated": 1e3 * s.T / value, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(s, a.gpus), "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(s, n):
    return {"workload": f"{s.name}_T{s.T}", "T_per_gpu": s.T, "H": s.H, "E": s.E, "K": s.K,
            "I": s.I, "I_shared": s.I_shared,
            "score_fn": ("softmax", "sigmoid", "sqrtsoftplus")[s.score_fn],
            "renorm": bool(s.renorm),
            "route_scale": s.route_scale, "global_tokens": s.T * n,
            "parallelism": f"replicas x{n}" if n > 1 else "single GPU",
            "l2": "inputs larger than L2 (expert weights and per-step intermediates exceed "
                  "126 MB), no flush"}


def time_extras(cfg, layer, x, b, moe, torch, hbm_gbs, tflops, reps=20):
    """The next-row calls on this step's tensors, each in its own loop of CUDA-event-timed
    launches: the order-invariant combine (against the rank-order one), the router
    statistics and the layer's backward. Their inputs come from the stage API once,
    outside the timing."""
    w = layer.w
    offsets, perm_token, dest_row, x_perm = moe.permute(cfg, b["topk_ids"], x=x)
    y, ys = moe.grouped_ffn(cfg, x, x_perm, perm_token, offsets, w["w13"], w["w2"],
                            w.get("w13_s"), w.get("w2_s"))
    del x_perm

    def loop(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # hold the stream while the calls are queued, so that the events time the device's
        # back-to-back work and not the host's launch rate
        torch.cuda.synchronize()
        torch.cuda._sleep(50_000_000)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    ref = moe.combine(cfg, y, b["topk_w"], dest_row, ys)
    inv = moe.combine(cfg, y, b["topk_w"], dest_row, ys, order_invariant=True)
    ms_c = loop(lambda: moe.combine(cfg, y, b["topk_w"], dest_row, ys))
    ms_i = loop(lambda: moe.combine(cfg, y, b["topk_w"], dest_row, ys, order_invariant=True))
    ms_s = loop(lambda: moe.router_stats(cfg, b["logits"], offsets))
    T, H, K, E = cfg.T, cfg.H, cfg.K, cfg.E

    # backward of the whole layer (moe_backward), dout synthetic
    from deterministic_invariant_routing_b200 import synthetic
    has_shared = ys is not None
    del y, ys
    dout = synthetic.normal_bf16(T, H, 1.0, 4242, "fill", device=x.device)
    ws = torch.empty(moe.workspace_bytes(cfg, moe.N.MOE_STAGE_BACKWARD), dtype=torch.uint8,
                     device=x.device)
    bwd = lambda: moe.backward(cfg, x, w["w_router"], w["w13"], w["w2"], b["logits"],  # noqa: E731
                               b["topk_ids"], b["topk_w"], dout, w13_s=w.get("w13_s"),
                               w2_s=w.get("w2_s"), ws=ws, check=False)
    ms_b = loop(bwd)
    # the training pair: moe_forward_train leaves the intermediates, the backward reuses them
    moe.forward_train(cfg, x, w["w_router"], w["w13"], w["w2"], ws, w13_s=w.get("w13_s"),
                      w2_s=w.get("w2_s"), logit_bias=w.get("logit_bias"),
                      sel_bias=w.get("sel_bias"))
    bwd_saved = lambda: moe.backward(cfg, x, w["w_router"], w["w13"], w["w2"],  # noqa: E731
                                     b["logits"], b["topk_ids"], b["topk_w"], dout,
                                     w13_s=w.get("w13_s"), w2_s=w.get("w2_s"), ws=ws,
                                     saved=True, check=False)
    ms_bs = loop(bwd_saved)
    fwd_train = lambda: moe.forward_train(cfg, x, w["w_router"], w["w13"], w["w2"], ws,  # noqa: E731
                                          w13_s=w.get("w13_s"), w2_s=w.get("w2_s"),
                                          logit_bias=w.get("logit_bias"),
                                          sel_bias=w.get("sel_bias"), check=False)
    ms_ft = loop(fwd_train)
    rows = int(offsets[-1].item())
    I, Is = cfg.I, cfg.I_shared
    # algorithmic: dh, dx rows, dW2, dW13 (12 H I per routed row), router dx and dW, shared
    bwd_flops = 12 * H * I * rows + 4 * T * H * E + 12 * T * H * Is
    # executed on top: the recomputed gate_up (twice) and down
    recompute_flops = 10 * H * I * rows + 6 * T * H * Is
    del ws
    comb_bytes = T * K * H * 2 + T * H * 2 + T * K * 8 + (T * H * 2 if has_shared else 0)
    stat_bytes = T * E * 4
    same = (ref.view(torch.int16) == inv.view(torch.int16)).float().mean().item()
    return {
        "combine_invariant": {"ms": ms_i, "rank_order_combine_ms": ms_c,
                              "achieved_gbs": comb_bytes / (ms_i * 1e-3) / 1e9,
                              "frac_hbm": comb_bytes / (ms_i * 1e-3) / 1e9 / hbm_gbs,
                              "algorithmic_bytes": comb_bytes,
                              "bits_equal_to_rank_order_fraction": same},
        "router_stats": {"ms": ms_s, "achieved_gbs": stat_bytes / (ms_s * 1e-3) / 1e9,
                         "frac_hbm": stat_bytes / (ms_s * 1e-3) / 1e9 / hbm_gbs,
                         "algorithmic_bytes": stat_bytes},
        "backward": {"ms": ms_b, "tokens_per_s": T / (ms_b * 1e-3),
                     "algorithmic_flops": bwd_flops,
                     "achieved_tflops": bwd_flops / (ms_b * 1e-3) / 1e12,
                     "frac_bf16_sustained": bwd_flops / (ms_b * 1e-3) / 1e12 / tflops,
                     "executed_flops_with_recompute": bwd_flops + recompute_flops,
                     "call": "moe_backward (dx, dW13, dW2, dW_router; forward intermediates "
                             "recomputed)",
                     "ms_with_saved_intermediates": ms_bs,
                     "frac_bf16_sustained_saved": bwd_flops / (ms_bs * 1e-3) / 1e12 / tflops,
                     "forward_train_ms": ms_ft,
                     "train_step_ms": ms_ft + ms_bs},
        "timing": f"CUDA events, {reps} back-to-back launches each, inputs of one bench step",
    }


BATCH_SWEEP = [1, 2, 3, 7, 16, 64, 255, 256, 1000, 2047, 2048, 2049, 4096, 8192, 16384]


def run_sweep(a):
    """Tokens/s of the layer forward at each batch size of the invariance sweep (the same
    batch sizes as the bit-equality tests), inputs resident in HBM. Between timed calls a
    256 MiB buffer is written so that small batches do not find their experts' weights in
    L2 from the previous call. One JSON object on stdout."""
    import torch

    from deterministic_invariant_routing_b200 import moe, synthetic

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    s = synthetic.shape(a.workload, T=max(BATCH_SWEEP))
    weights = synthetic.make_weights(s, device=dev)
    x_all = synthetic.make_tokens(s, s.T, seed=s.seed + 5, device=dev)
    cfg = moe.Config.of(s)
    layer = moe.MoELayer(cfg, weights)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rows = []
    for B in BATCH_SWEEP:
        x = x_all[:B].contiguous()
        for _ in range(3):
            layer(x, check=False)
        reps = 50 if B < 4096 else 20
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            layer(x, check=False)
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        moe.check_status(layer.status)
        ms = statistics.median(ts)
        rows.append({"B": B, "ms": ms, "tokens_per_s": B / (ms * 1e-3)})
    print(json.dumps({"sweep": f"{s.name} layer forward by batch size", "l2": "256 MiB "
                      "written between calls", "timing": "median of CUDA-event-timed calls",
                      "rows": rows}), flush=True)


def run_oracle_sweep(a):
    """The oracle's layer forward on the host cores for each workload: tokens/s on a bounded
    token sample (about 3 s each), with the host's core count and CPU model."""
    import platform

    import torch

    from deterministic_invariant_routing_b200 import synthetic

    import oracle
    gen = "cuda" if torch.cuda.is_available() else "cpu"  # weights drawn on the GPU if any
    model = platform.processor()
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    cases = [("tiny", 64), ("dspark", 8192), ("qwen3_30b_a3b", 1), ("qwen3_30b_a3b", 64),
             ("qwen3_30b_a3b", 4096), ("qwen3_30b_a3b", 16384), ("dsv_sigmoid", 8192)]
    rows = []
    for name, T in cases:
        s, d = synthetic.make_layer(name, T=T, device=gen)
        d = {k: (None if v is None else v.cpu()) for k, v in d.items()}
        r = cpu_baseline(s, d, seconds=3.0)
        del d
        rows.append({"workload": f"{name}_T{T}", "tokens_per_s": r["value"],
                     "sample": r["sample"]})
    print(json.dumps({"oracle_sweep": "oracle layer forward on the host cores",
                      "nproc": os.cpu_count(), "threads": oracle.num_threads(),
                      "cpu_model": model, "rows": rows}), flush=True)


def main():
    a = parse()
    if a.impl == "reference":
        return run_reference(a)
    if a.sweep:
        return run_sweep(a)
    if a.oracle_sweep:
        return run_oracle_sweep(a)

    import torch
    import torch.distributed as dist

    from deterministic_invariant_routing_b200 import moe, synthetic

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    s = synthetic.shape(a.workload, T=a.T)
    weights, x = replica_inputs(s, rank, dev)
    cfg = moe.Config.of(s)
    layer = moe.MoELayer(cfg, weights)

    for _ in range(a.warmup):
        layer(x, check=False)
    out, b = layer(x, keep=True, check=True)  # fail closed once before timing
    offsets = b["offsets"].cpu()
    n_touched = int(((offsets[1:] - offsets[:-1]) > 0).sum())
    rows = int(offsets[-1])

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(v):
        return reduce_max(v, dev, world)

    K = a.steps
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    barrier()
    with ClockSampler(gpu_id) as clk:
        start.record()
        for k in range(K):
            layer(x, check=False)
        stop.record()
        barrier()
    ms = max_over_ranks(start.elapsed_time(stop) / K)
    moe.check_status(layer.status)

    # the stage split, in a separate pass: events recorded between the kernels break the
    # dependent-launch overlap, so they stay out of the timed steps above
    Ks = max(1, min(a.split_steps, K))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(Ks)]
    for k in range(Ks):
        layer(x, check=False, stage_events=ev[k])
    barrier()
    moe.check_status(layer.status)

    def stage_ms(i, j):
        return statistics.fmean(e[i].elapsed_time(e[j]) for e in ev)

    stages = {"router_gemm": stage_ms(0, 1), "route": stage_ms(1, 2), "dispatch": stage_ms(2, 3),
              "gate_up_gemm": stage_ms(3, 4), "down_gemm": stage_ms(4, 5),
              "shared_expert": stage_ms(5, 6), "combine": stage_ms(6, 7)}

    # end to end through the C-ABI call on host buffers (moe_forward_host): every step
    # copies x from pinned host memory and the output back, overlapped chunk by chunk
    Ke = a.e2e_steps or K
    x_h = x.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    for _ in range(3):
        layer.forward_host(x_h, out_h, chunk=a.e2e_chunk, check=False)
    moe.check_status(layer.status)
    if not torch.equal(out_h.view(torch.int16), out.cpu().view(torch.int16)):
        raise RuntimeError("host-memory path differs from the device path")
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(Ke):
        layer.forward_host(x_h, out_h, chunk=a.e2e_chunk, check=False)
    e1.record()
    barrier()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1) / Ke)
    moe.check_status(layer.status)

    pk, pk_src = peaks()
    flops, byts = layer_work(s, n_touched)
    # the peak that applies: a timed region shorter than about a second runs at the boost
    # clock (the burst peak); a longer one settles under the power cap (the sustained one)
    busy_ms = ms * (K + Ks)
    regime = "sustained" if busy_ms >= 1000.0 else "burst"
    peak_of = {"burst": pk["bf16_tflops"], "sustained": pk["bf16_tflops_sustained"]}
    peak = peak_of[regime]
    gate_ms = max_over_ranks(stages["gate_up_gemm"])
    gate_flops = 4 * rows * s.H * s.I
    # the kernel's own operands read once and its result written once
    gate_bytes = n_touched * 2 * s.I * s.H * 2 + rows * s.H * 2 + rows * s.I * 2
    t_flop = gate_flops / (peak * 1e12)
    t_byte = gate_bytes / (pk["hbm_gbs"] * 1e9)
    if t_flop >= t_byte:
        bound, work, unit, pk_k = "tensor", gate_flops, "TFLOP/s", peak
        achieved = gate_flops / (gate_ms * 1e-3) / 1e12
        fracs = {f"frac_{r}": achieved / v for r, v in peak_of.items()}
        pk_desc = f"{pk_src} bf16 {regime}"
    else:
        bound, work, unit, pk_k = "hbm", gate_bytes, "GB/s", pk["hbm_gbs"]
        achieved = gate_bytes / (gate_ms * 1e-3) / 1e9
        fracs = {}
        pk_desc = f"{pk_src} HBM copy"
    t_roof = {r: max(flops / (v * 1e12), byts / (pk["hbm_gbs"] * 1e9))
              for r, v in peak_of.items()}
    clocks = clk.summary()
    line = {
        "metric": "MoE-layer tokens/s (bf16, batch-invariant)",
        "value": job_tokens_per_s(s.T, world, ms), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(s, world),
        "roofline": {"bound": bound, "kernel": "gate_up grouped GEMM + SwiGLU (tcgen05)",
                     "achieved": achieved, "peak": pk_k, "unit": unit,
                     "frac": achieved / pk_k, **fracs,
                     "traffic": ncu_traffic("gate_up", rows, s.name, f"{s.name}_T{s.T}"),
                     "peak_source": pk_desc, "peak_regime": regime,
                     "regime_rule": "burst when the timed steps plus the stage-split pass "
                                    f"keep the GPU busy under 1 s (here {busy_ms:.0f} ms)",
                     "algorithmic_flops_per_launch": gate_flops,
                     "algorithmic_bytes_per_launch": gate_bytes,
                     "kernel_ms": gate_ms},
        "layer_roofline": {"flops": flops, "bytes": byts, "roofline_ms": t_roof[regime] * 1e3,
                           "frac": t_roof[regime] * 1e3 / ms,
                           "frac_burst": t_roof["burst"] * 1e3 / ms,
                           "frac_sustained": t_roof["sustained"] * 1e3 / ms,
                           "experts_touched": n_touched, "routed_rows": rows,
                           "peaks": f"{pk_src}: {pk['bf16_tflops']} TFLOP/s bf16 burst, "
                                    f"{pk['bf16_tflops_sustained']} sustained, "
                                    f"{pk['hbm_gbs']} GB/s; {regime} applies"},
        "stage_ms": stages,
        "stage_split": f"separate pass of {Ks} steps with events between the kernels "
                       f"({sum(stages.values()):.4f} ms per step there)",
        "e2e": {"value": job_tokens_per_s(s.T, world, ms_e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": out.numel() * 2,
                "ms_per_step": ms_e2e, "chunk_tokens": a.e2e_chunk,
                "call": "moe_forward_host (pinned host in/out, copies overlapped)"},
        "gpu_launches": K * (10 + (3 if s.I_shared else 0)),
        "clocks": clocks,
    }
    if not a.no_extras:
        line["extras"] = time_extras(cfg, layer, x, b, moe, torch, pk["hbm_gbs"],
                                     pk["bf16_tflops_sustained"], reps=a.extras_reps)
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        d_cpu = {k: (None if v is None else v.cpu()) for k, v in weights.items()}
        d_cpu["x"] = x.cpu()
        line["cpu_baseline"] = cpu_baseline(s, d_cpu)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Shared helpers of the GPU tests: building layers on the device, reference values from
the oracle for sampled tokens, and the error metrics of the parity levels."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from deterministic_invariant_routing_b200 import moe, synthetic

DEV = "cuda:0"

# Level-2 bar: per token row, max|gpu - ref| / max|ref| (bf16 output vs the FP64 layer)
LEVEL2_ROW_REL = 1e-2


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bits of a tensor as an unsigned numpy array (bf16 -> uint16, fp32 -> uint32)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    return t.numpy()


def layer(name: str, T=None, device=DEV, **over):
    s, d = synthetic.make_layer(name, T=T, device=device, **over)
    return s, d, moe.Config.of(s)


def expert_subset(d, ids_rows: np.ndarray):
    """CPU copies of only the experts that the given routes use, and the routes remapped
    onto that subset (keeps oracle inputs small for layers with GBs of weights)."""
    used = np.unique(ids_rows[ids_rows >= 0])
    remap = np.full(int(d["w13"].shape[0]), -1, np.int32)
    remap[used] = np.arange(used.size, dtype=np.int32)
    sel = torch.from_numpy(used.astype(np.int64)).to(d["w13"].device)
    w13 = d["w13"].index_select(0, sel).cpu()
    w2 = d["w2"].index_select(0, sel).cpu()
    ids_sub = np.where(ids_rows >= 0, remap[np.maximum(ids_rows, 0)], -1).astype(np.int32)
    return w13, w2, ids_sub


def reference_rows(s, d, x_rows_cpu, logits64_rows, ids_rows, mask_rows=None):
    """FP64 layer output of some tokens for the given routes (the FP32-contract routes),
    with weights recomputed in FP64 from FP64 scores."""
    w64 = oracle.weights64(logits64_rows, ids_rows, s.score_fn, s.renorm, s.route_scale)
    w13, w2, ids_sub = expert_subset(d, ids_rows)
    w13s = d["w13_s"].cpu() if d.get("w13_s") is not None else None
    w2s = d["w2_s"].cpu() if d.get("w2_s") is not None else None
    return oracle.forward64(x_rows_cpu, ids_sub, w64, w13, w2, w13s, w2s, mask=mask_rows)


def row_rel_err(gpu_bf16: torch.Tensor, ref64: np.ndarray) -> np.ndarray:
    g = gpu_bf16.detach().float().cpu().numpy().astype(np.float64)
    den = np.maximum(np.abs(ref64).max(axis=1), 1e-30)
    return np.abs(g - ref64).max(axis=1) / den


def mean_abs_err(gpu_bf16: torch.Tensor, ref64: np.ndarray) -> float:
    g = gpu_bf16.detach().float().cpu().numpy().astype(np.float64)
    return float(np.abs(g - ref64).mean())


def near_tie_count(logits_f32: np.ndarray, s, sel_bias=None) -> int:
    """Tokens whose K-th and (K+1)-th selection choices are within 1 fp32 ulp (by the
    oracle's contract scores)."""
    if s.K >= s.E:
        return 0
    n = 0
    b = None if sel_bias is None else np.asarray(sel_bias, np.float32)
    for row in logits_f32:
        sc = oracle.scores_fp32(row, s.score_fn)
        c = sc if b is None else (sc + b).astype(np.float32)
        c = c[~np.isnan(c)]
        if c.size <= s.K:
            continue
        top = np.sort(c)[::-1]
        a, z = np.float32(top[s.K - 1]), np.float32(top[s.K])
        if a - z <= np.spacing(a):
            n += 1
    return n

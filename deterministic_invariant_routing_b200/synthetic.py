"""Seeded synthetic inputs for the MoE FFN layer, shared by the tests, the bench and smoke().

This module only draws random numbers and shapes them; it computes nothing of the
method itself (no scores, no routing, no expert math).  Both the CUDA path and the
oracle receive the tensors made here.

Workload shapes follow the layers the source pages talk about:

* ``tiny``: a toy layer for fast checks (hidden 128, 8 experts x 256, top-2).
* ``dspark``: the DSpark draft FFN of the SpecForge MoE-draft PR (8 experts x 1536,
  top-1 without renormalisation, softmax scores, selection bias) -- SpecForge PR #1003,
  "Verification" and the draft-config commit.
* ``qwen3_30b_a3b``: a Qwen3-30B-A3B-shaped layer (hidden 2048, 128 experts x 768,
  top-8, softmax, renormalised), the model of the UniRL parity PR (#430, "Supported
  case"); an expert logit bias skews the loads.
* ``dsv_sigmoid``: a DeepSeek-style sigmoid router layer (256 experts x 1024, top-6,
  selection bias, route_scale 2.5, one always-on shared expert of width 2048) -- the
  DeepSeek seams named in SpecForge PR #1003, "Out of scope".

Every tensor gets its own generator seeded from (workload seed, tensor tag), so a
tensor does not depend on which other tensors were drawn or in what order, and the
token rows of ``x`` for a given seed do not depend on the batch they are placed in.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

SOFTMAX = 0
SIGMOID = 1
SQRTSOFTPLUS = 2


@dataclasses.dataclass(frozen=True)
class LayerShape:
    name: str
    T: int
    H: int
    E: int
    I: int
    K: int
    score_fn: int
    renorm: bool
    route_scale: float
    I_shared: int
    x_std: float
    w_std: float
    sel_bias_range: Optional[float]   # selection bias ~ U(-r, r), or None
    logit_bias_std: Optional[float]   # per-expert logit skew ~ N(0, s), or None
    seed: int
    n_group: int = 0                  # group-limited selection (0 = off)
    topk_group: int = 0


WORKLOADS = {
    "tiny": LayerShape("tiny", T=64, H=128, E=8, I=256, K=2, score_fn=SOFTMAX, renorm=True,
                       route_scale=1.0, I_shared=0, x_std=0.02, w_std=0.02,
                       sel_bias_range=None, logit_bias_std=None, seed=1),
    "dspark": LayerShape("dspark", T=8192, H=4096, E=8, I=1536, K=1, score_fn=SOFTMAX,
                         renorm=False, route_scale=1.0, I_shared=0, x_std=1.0, w_std=0.02,
                         sel_bias_range=0.05, logit_bias_std=None, seed=2),
    "qwen3_30b_a3b": LayerShape("qwen3_30b_a3b", T=16384, H=2048, E=128, I=768, K=8,
                                score_fn=SOFTMAX, renorm=True, route_scale=1.0, I_shared=0,
                                x_std=1.0, w_std=0.02, sel_bias_range=None,
                                logit_bias_std=0.5, seed=3),
    "dsv_sigmoid": LayerShape("dsv_sigmoid", T=8192, H=4096, E=256, I=1024, K=6,
                              score_fn=SIGMOID, renorm=True, route_scale=2.5, I_shared=2048,
                              x_std=1.0, w_std=0.02, sel_bias_range=0.05,
                              logit_bias_std=None, seed=4),
}

# tags keep every tensor's stream independent of the others
_TAG = {"x": 1, "w_router": 2, "logit_bias": 3, "sel_bias": 4, "w13": 5, "w2": 6,
        "w13_s": 7, "w2_s": 8, "mask": 9, "perm": 10, "logits": 11, "fill": 12}


def shape(name: str, **overrides) -> LayerShape:
    return dataclasses.replace(WORKLOADS[name], **overrides)


def _gen(seed: int, tag: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + _TAG[tag] * 7919)
    return g


def normal_bf16(rows: int, cols: int, std: float, seed: int, tag: str, device="cpu",
                batch: int = 0) -> torch.Tensor:
    """bf16 draws of N(0, std^2): an fp32 normal draw, scaled, rounded to nearest even."""
    g = _gen(seed, tag, device)
    size = (batch, rows, cols) if batch else (rows, cols)
    v = torch.randn(size, generator=g, device=device, dtype=torch.float32)
    return (v * std).to(torch.bfloat16)


def uniform_f32(n: int, lim: float, seed: int, tag: str, device="cpu") -> torch.Tensor:
    g = _gen(seed, tag, device)
    return (torch.rand(n, generator=g, device=device, dtype=torch.float32) * 2.0 - 1.0) * lim


def make_tokens(s: LayerShape, T: int, seed: Optional[int] = None, device="cpu",
                tag: str = "x") -> torch.Tensor:
    """T token rows of the workload's activation distribution."""
    return normal_bf16(T, s.H, s.x_std, s.seed if seed is None else seed, tag, device)


def make_weights(s: LayerShape, device="cpu") -> dict:
    """Router, expert and shared-expert weights of the layer (random init, no checkpoint).

    Layouts: w_router [E,H]; w13 [E, 2I, H] with the I gate rows first, then the I up
    rows (both K-major, i.e. rows of length H); w2 [E, H, I]; the shared expert the same
    with I_shared and no expert axis.
    """
    d = {
        "w_router": normal_bf16(s.E, s.H, s.w_std, s.seed, "w_router", device),
        "w13": normal_bf16(2 * s.I, s.H, s.w_std, s.seed, "w13", device, batch=s.E),
        "w2": normal_bf16(s.H, s.I, s.w_std, s.seed, "w2", device, batch=s.E),
        "logit_bias": None,
        "sel_bias": None,
        "w13_s": None,
        "w2_s": None,
    }
    if s.logit_bias_std is not None:
        g = _gen(s.seed, "logit_bias", device)
        d["logit_bias"] = torch.randn(s.E, generator=g, device=device) * s.logit_bias_std
    if s.sel_bias_range is not None:
        d["sel_bias"] = uniform_f32(s.E, s.sel_bias_range, s.seed, "sel_bias", device)
    if s.I_shared:
        d["w13_s"] = normal_bf16(2 * s.I_shared, s.H, s.w_std, s.seed, "w13_s", device)
        d["w2_s"] = normal_bf16(s.H, s.I_shared, s.w_std, s.seed, "w2_s", device)
    return d


def make_layer(name: str, T: Optional[int] = None, device="cpu", **overrides) -> tuple:
    """(shape, inputs) for a named workload; inputs holds x plus make_weights()."""
    s = shape(name, **overrides)
    if T is not None:
        s = dataclasses.replace(s, T=T)
    d = make_weights(s, device)
    d["x"] = make_tokens(s, s.T, device=device)
    return s, d


def random_logits(T: int, E: int, seed: int, std: float = 1.0, device="cpu") -> torch.Tensor:
    """fp32 router logits for routing-only checks (the logits-in mode)."""
    g = _gen(seed, "logits", device)
    return torch.randn(T, E, generator=g, device=device) * std


def random_mask(T: int, keep: float, seed: int) -> torch.Tensor:
    """uint8 token mask, 1 = a real token, 0 = padding."""
    g = _gen(seed, "mask", "cpu")
    return (torch.rand(T, generator=g) < keep).to(torch.uint8)


def random_permutation(n: int, seed: int) -> torch.Tensor:
    g = _gen(seed, "perm", "cpu")
    return torch.randperm(n, generator=g)


def bf16_bits(t: torch.Tensor):
    """A bf16 tensor as a numpy uint16 array of its raw bits (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")

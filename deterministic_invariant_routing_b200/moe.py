"""Python binding of libmoe_b200: torch tensors in, the C ABI's calls out.

Argument marshalling only -- shapes, dtypes and devices are checked, buffers are
allocated with torch (device memory is torch's), and every step of the layer runs in
the library's CUDA kernels on torch's current stream. Calls fail closed: a nonzero
return code raises ``MoeError``; with ``check=True`` the stream is synchronised and a
nonzero device status word (NaN scores, zero renormalisation denominator, bad expert
id, pipeline timeout) raises ``StatusError`` ("DSV4 Flash MoE Train-Inference
Consistency Roadmap", Follow-Up Issue Buckets: mismatches fail closed; UniRL PR #430:
abort rather than continue on a parity failure).
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional, Sequence

import torch

from . import _native as N

SOFTMAX = N.MOE_SOFTMAX
SIGMOID = N.MOE_SIGMOID
SQRTSOFTPLUS = N.MOE_SQRTSOFTPLUS
STATUS_NAMES = ("nan_tokens", "zero_denominator", "bad_expert_id", "pipeline_timeout")


class MoeError(RuntimeError):
    pass


class StatusError(MoeError):
    def __init__(self, words):
        self.words = list(words)
        named = {n: w for n, w in zip(STATUS_NAMES, self.words) if w}
        super().__init__(f"device status reports anomalies: {named}")


@dataclasses.dataclass(frozen=True)
class Config:
    T: int
    H: int
    E: int
    K: int
    I: int
    I_shared: int = 0
    score_fn: int = SOFTMAX
    renorm: bool = True
    route_scale: float = 1.0
    n_group: int = 0        # group-limited selection, 0 = off
    topk_group: int = 0

    @classmethod
    def of(cls, shape, T: Optional[int] = None) -> "Config":
        """From a workload shape (anything with the same field names)."""
        return cls(T=shape.T if T is None else T, H=shape.H, E=shape.E, K=shape.K, I=shape.I,
                   I_shared=shape.I_shared, score_fn=shape.score_fn, renorm=bool(shape.renorm),
                   route_scale=float(shape.route_scale),
                   n_group=int(getattr(shape, "n_group", 0)),
                   topk_group=int(getattr(shape, "topk_group", 0)))

    def with_T(self, T: int) -> "Config":
        return dataclasses.replace(self, T=T)

    def c(self) -> N.MoeCfg:
        return N.MoeCfg(self.T, self.H, self.E, self.K, self.I, self.I_shared, self.score_fn,
                        int(bool(self.renorm)), float(self.route_scale), int(self.n_group),
                        int(self.topk_group))


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need(t, name, dtype, shape, dev):
    if t is None:
        raise MoeError(f"{name} is required")
    if t.dtype != dtype:
        raise MoeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise MoeError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.device != dev:
        raise MoeError(f"{name}: on {t.device}, expected {dev}")
    if not t.is_contiguous():
        raise MoeError(f"{name} must be contiguous")
    return t


def _opt(t, name, dtype, shape, dev):
    return None if t is None else _need(t, name, dtype, shape, dev)


def _rc(code: int, what: str):
    if code != N.MOE_OK:
        raise MoeError(f"{what}: {N.status_string(code)} ({code})")


def workspace_bytes(cfg: Config, stage: int) -> int:
    return int(N.load().moe_workspace_bytes(ctypes.byref(cfg.c()), stage))


def new_status(dev) -> torch.Tensor:
    return torch.zeros(N.MOE_STATUS_WORDS, dtype=torch.int32, device=dev)


def check_status(status: torch.Tensor, stream_sync: bool = True):
    if stream_sync:
        torch.cuda.current_stream(status.device).synchronize()
    words = status.cpu().tolist()
    if any(words):
        raise StatusError(words)


def _ws(nbytes: int, dev, ws: Optional[torch.Tensor]) -> torch.Tensor:
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise MoeError(f"workspace of {ws.numel() * ws.element_size()} bytes < {nbytes}")
        return ws
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)


# ------------------------------------------------------------------ stages

def route(cfg: Config, x=None, w_router=None, logits=None, logit_bias=None, sel_bias=None,
          token_mask=None, status=None, check: bool = True):
    """Routing boundary. With x: logits are computed (returned); with x=None the given
    fp32 logits [T,E] are routed. Returns (logits, topk_ids, topk_w)."""
    dev = (x if x is not None else logits).device
    T, H, E, K = cfg.T, cfg.H, cfg.E, cfg.K
    if x is not None:
        _need(x, "x", torch.bfloat16, (T, H), dev)
        _need(w_router, "w_router", torch.bfloat16, (E, H), dev)
        logits = torch.empty(T, E, dtype=torch.float32, device=dev) if logits is None else logits
    _need(logits, "logits", torch.float32, (T, E), dev)
    _opt(logit_bias, "logit_bias", torch.float32, (E,), dev)
    _opt(sel_bias, "sel_bias", torch.float32, (E,), dev)
    _opt(token_mask, "token_mask", torch.uint8, (T,), dev)
    ids = torch.empty(T, K, dtype=torch.int32, device=dev)
    w = torch.empty(T, K, dtype=torch.float32, device=dev)
    st = new_status(dev) if status is None else status
    _rc(N.load().moe_route(ctypes.byref(cfg.c()), _p(x), _p(w_router), _p(logit_bias),
                           _p(sel_bias), _p(token_mask), _p(logits), _p(ids), _p(w), _p(st),
                           _stream(dev)), "moe_route")
    if check:
        check_status(st)
    return logits, ids, w


def permute(cfg: Config, topk_ids, x=None, want_x_perm: bool = True, status=None,
            check: bool = True):
    """Dispatch boundary. Returns (offsets [E+1], perm_token [T*K], dest_row [T,K],
    x_perm [T*K,H] or None)."""
    dev = topk_ids.device
    T, K, E, H = cfg.T, cfg.K, cfg.E, cfg.H
    _need(topk_ids, "topk_ids", torch.int32, (T, K), dev)
    _opt(x, "x", torch.bfloat16, (T, H), dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm_token = torch.full((T * K,), -1, dtype=torch.int32, device=dev)
    dest_row = torch.empty(T, K, dtype=torch.int32, device=dev)
    x_perm = None
    if want_x_perm and x is not None:
        x_perm = torch.empty(T * K, H, dtype=torch.bfloat16, device=dev)
    nbytes = workspace_bytes(cfg, N.MOE_STAGE_PERMUTE)
    ws = _ws(nbytes, dev, None)
    st = new_status(dev) if status is None else status
    _rc(N.load().moe_permute(ctypes.byref(cfg.c()), _p(topk_ids), _p(x), _p(offsets),
                             _p(perm_token), _p(dest_row), _p(x_perm), _p(st), _p(ws),
                             ws.numel(), _stream(dev)), "moe_permute")
    if check:
        check_status(st)
    return offsets, perm_token, dest_row, x_perm


def grouped_ffn(cfg: Config, x, x_perm, perm_token, offsets, w13, w2, w13_s=None, w2_s=None,
                status=None, check: bool = True):
    """Expert boundary. Returns (y [T*K,H], y_shared [T,H] or None)."""
    dev = offsets.device
    T, H, E, K, I, Is = cfg.T, cfg.H, cfg.E, cfg.K, cfg.I, cfg.I_shared
    _opt(x, "x", torch.bfloat16, (T, H), dev)
    _opt(x_perm, "x_perm", torch.bfloat16, (T * K, H), dev)
    _opt(perm_token, "perm_token", torch.int32, (T * K,), dev)
    _need(offsets, "offsets", torch.int32, (E + 1,), dev)
    _need(w13, "w13", torch.bfloat16, (E, 2 * I, H), dev)
    _need(w2, "w2", torch.bfloat16, (E, H, I), dev)
    if Is:
        _need(w13_s, "w13_s", torch.bfloat16, (2 * Is, H), dev)
        _need(w2_s, "w2_s", torch.bfloat16, (H, Is), dev)
    y = torch.empty(T * K, H, dtype=torch.bfloat16, device=dev)
    y_s = torch.empty(T, H, dtype=torch.bfloat16, device=dev) if Is else None
    ws = _ws(workspace_bytes(cfg, N.MOE_STAGE_FFN), dev, None)
    st = new_status(dev) if status is None else status
    _rc(N.load().moe_grouped_ffn(ctypes.byref(cfg.c()), _p(x), _p(x_perm), _p(perm_token),
                                 _p(offsets), _p(w13), _p(w2), _p(w13_s), _p(w2_s), _p(y),
                                 _p(y_s), _p(st), _p(ws), ws.numel(), _stream(dev)),
        "moe_grouped_ffn")
    if check:
        check_status(st)
    return y, y_s


def combine(cfg: Config, y, topk_w, dest_row, y_shared=None, token_mask=None,
            order_invariant: bool = False):
    """Reduction boundary. Returns out [T,H] bf16. order_invariant=True runs the
    canonical-order variant (moe_combine_invariant) instead of the rank-order contract."""
    dev = y.device
    T, H, K = cfg.T, cfg.H, cfg.K
    if y.dim() != 2 or y.shape[1] != H or y.dtype != torch.bfloat16 or not y.is_contiguous():
        raise MoeError("y must be a contiguous bf16 [rows, H] tensor")
    _need(topk_w, "topk_w", torch.float32, (T, K), dev)
    _need(dest_row, "dest_row", torch.int32, (T, K), dev)
    _opt(y_shared, "y_shared", torch.bfloat16, (T, H), dev)
    _opt(token_mask, "token_mask", torch.uint8, (T,), dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    fn = N.load().moe_combine_invariant if order_invariant else N.load().moe_combine
    _rc(fn(ctypes.byref(cfg.c()), _p(y), _p(topk_w), _p(dest_row), _p(y_shared),
           _p(token_mask), _p(out), _stream(dev)), "moe_combine")
    return out


def pipeline_wait_selftest(dev, limit_cycles: int = 1_000_000, check: bool = True):
    """Run one bounded pipeline wait that nothing satisfies (moe_pipeline_wait_selftest):
    it gives up after limit_cycles and counts a pipeline timeout in the returned status
    words; with check=True the count raises StatusError, as in any other call."""
    st = new_status(dev)
    _rc(N.load().moe_pipeline_wait_selftest(_p(st), int(limit_cycles), _stream(st.device)),
        "moe_pipeline_wait_selftest")
    if check:
        check_status(st)
    return st


def router_stats(cfg: Config, logits, offsets, token_mask=None):
    """Router statistics of a routed batch: {tokens_per_expert [E] int32, mean_prob [E]
    fp32, aux [1] fp32} (the load-balance value E * sum_e load_e * mean_prob_e, K when
    balanced). logits and offsets as returned by route()/permute() or forward(keep=True)."""
    dev = logits.device
    T, E = cfg.T, cfg.E
    _need(logits, "logits", torch.float32, (T, E), dev)
    _need(offsets, "offsets", torch.int32, (E + 1,), dev)
    _opt(token_mask, "token_mask", torch.uint8, (T,), dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    mp = torch.empty(E, dtype=torch.float32, device=dev)
    aux = torch.empty(1, dtype=torch.float32, device=dev)
    ws = _ws(workspace_bytes(cfg, N.MOE_STAGE_STATS), dev, None)
    _rc(N.load().moe_router_stats(ctypes.byref(cfg.c()), _p(logits), _p(token_mask),
                                  _p(offsets), _p(counts), _p(mp), _p(aux), _p(ws), ws.numel(),
                                  _stream(dev)), "moe_router_stats")
    return {"tokens_per_expert": counts, "mean_prob": mp, "aux": aux}


# ------------------------------------------------------------------ backward

def backward_workspace(cfg: Config, dev) -> torch.Tensor:
    """A workspace for forward_train() + backward(saved=True) (or backward alone)."""
    return _ws(workspace_bytes(cfg, N.MOE_STAGE_BACKWARD), dev, None)


def forward_train(cfg: Config, x, w_router, w13, w2, ws, logit_bias=None, sel_bias=None,
                  token_mask=None, w13_s=None, w2_s=None, status=None, check: bool = True):
    """The forward of a training step (moe_forward_train): the same output as forward(), and
    the intermediates the backward needs left in `ws` (backward_workspace()). Returns
    (out [T,H] bf16, {logits, topk_ids, topk_w}); then backward(..., ws=ws, saved=True)."""
    dev = x.device
    T, H, E, K, I, Is = cfg.T, cfg.H, cfg.E, cfg.K, cfg.I, cfg.I_shared
    _need(x, "x", torch.bfloat16, (T, H), dev)
    _need(w_router, "w_router", torch.bfloat16, (E, H), dev)
    _need(w13, "w13", torch.bfloat16, (E, 2 * I, H), dev)
    _need(w2, "w2", torch.bfloat16, (E, H, I), dev)
    _opt(logit_bias, "logit_bias", torch.float32, (E,), dev)
    _opt(sel_bias, "sel_bias", torch.float32, (E,), dev)
    _opt(token_mask, "token_mask", torch.uint8, (T,), dev)
    if Is:
        _need(w13_s, "w13_s", torch.bfloat16, (2 * Is, H), dev)
        _need(w2_s, "w2_s", torch.bfloat16, (H, Is), dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    b = {"logits": torch.empty(T, E, dtype=torch.float32, device=dev),
         "topk_ids": torch.empty(T, K, dtype=torch.int32, device=dev),
         "topk_w": torch.empty(T, K, dtype=torch.float32, device=dev)}
    nbytes = workspace_bytes(cfg, N.MOE_STAGE_BACKWARD)
    ws = _ws(nbytes, dev, ws)
    st = new_status(dev) if status is None else status
    _rc(N.load().moe_forward_train(ctypes.byref(cfg.c()), _p(x), _p(w_router), _p(logit_bias),
                                   _p(sel_bias), _p(token_mask), _p(w13), _p(w2), _p(w13_s),
                                   _p(w2_s), _p(out), _p(b["logits"]), _p(b["topk_ids"]),
                                   _p(b["topk_w"]), _p(st), _p(ws), nbytes, _stream(dev)),
        "moe_forward_train")
    if check:
        check_status(st)
    return out, b


def backward(cfg: Config, x, w_router, w13, w2, logits, topk_ids, topk_w, dout, token_mask=None,
             w13_s=None, w2_s=None, ws=None, status=None, keep: bool = False,
             saved: bool = False, check: bool = True) -> dict:
    """Gradients of sum(dout * out) of the layer for the forward's routes (moe_backward):
    {dx [T,H] bf16, dw_router [E,H], dw13 [E,2I,H], dw2 [E,H,I] fp32 (+ dw13_s, dw2_s with a
    shared expert)}; keep=True adds d_topk_w [T,K] and dlogits [T,E] (fp32).
    logits, topk_ids, topk_w: as forward(keep=True) or forward_train() returned them.
    saved=True: ws holds forward_train()'s intermediates for the same inputs (no recompute)."""
    if saved and ws is None:
        raise MoeError("saved=True needs the workspace forward_train() wrote")
    dev = x.device
    T, H, E, K, I, Is = cfg.T, cfg.H, cfg.E, cfg.K, cfg.I, cfg.I_shared
    _need(x, "x", torch.bfloat16, (T, H), dev)
    _need(w_router, "w_router", torch.bfloat16, (E, H), dev)
    _need(w13, "w13", torch.bfloat16, (E, 2 * I, H), dev)
    _need(w2, "w2", torch.bfloat16, (E, H, I), dev)
    _need(logits, "logits", torch.float32, (T, E), dev)
    _need(topk_ids, "topk_ids", torch.int32, (T, K), dev)
    _need(topk_w, "topk_w", torch.float32, (T, K), dev)
    _need(dout, "dout", torch.bfloat16, (T, H), dev)
    _opt(token_mask, "token_mask", torch.uint8, (T,), dev)
    if Is:
        _need(w13_s, "w13_s", torch.bfloat16, (2 * Is, H), dev)
        _need(w2_s, "w2_s", torch.bfloat16, (H, Is), dev)
    g = {"dx": torch.empty(T, H, dtype=torch.bfloat16, device=dev),
         "dw_router": torch.empty(E, H, dtype=torch.float32, device=dev),
         "dw13": torch.empty(E, 2 * I, H, dtype=torch.float32, device=dev),
         "dw2": torch.empty(E, H, I, dtype=torch.float32, device=dev),
         "dw13_s": torch.empty(2 * Is, H, dtype=torch.float32, device=dev) if Is else None,
         "dw2_s": torch.empty(H, Is, dtype=torch.float32, device=dev) if Is else None}
    if keep:
        g["d_topk_w"] = torch.empty(T, K, dtype=torch.float32, device=dev)
        g["dlogits"] = torch.empty(T, E, dtype=torch.float32, device=dev)
    nbytes = workspace_bytes(cfg, N.MOE_STAGE_BACKWARD)
    ws = _ws(nbytes, dev, ws)
    st = new_status(dev) if status is None else status
    _rc(N.load().moe_backward(ctypes.byref(cfg.c()), _p(x), _p(w_router), _p(token_mask),
                              _p(w13), _p(w2), _p(w13_s), _p(w2_s), _p(logits), _p(topk_ids),
                              _p(topk_w), _p(dout), _p(g["dx"]), _p(g["dw_router"]),
                              _p(g["dw13"]), _p(g["dw2"]), _p(g["dw13_s"]), _p(g["dw2_s"]),
                              _p(g.get("d_topk_w")), _p(g.get("dlogits")), int(bool(saved)),
                              _p(st), _p(ws), nbytes, _stream(dev)), "moe_backward")
    if check:
        check_status(st)
    return g


# ------------------------------------------------------------------ whole layer

def forward(cfg: Config, x, w_router, w13, w2, logit_bias=None, sel_bias=None, token_mask=None,
            w13_s=None, w2_s=None, out=None, ws=None, status=None, keep: bool = False,
            stage_events: Optional[Sequence] = None, check: bool = True):
    """The MoE layer (routing -> dispatch -> experts -> combine) in one C-ABI call.

    keep=True also returns the boundary tensors {logits, topk_ids, topk_w, offsets}.
    stage_events: MOE_NUM_STAGE_EVENTS torch.cuda.Event(enable_timing=True) recorded at
    the stage boundaries (for timing)."""
    dev = x.device
    T, H, E, K, I, Is = cfg.T, cfg.H, cfg.E, cfg.K, cfg.I, cfg.I_shared
    _need(x, "x", torch.bfloat16, (T, H), dev)
    _need(w_router, "w_router", torch.bfloat16, (E, H), dev)
    _need(w13, "w13", torch.bfloat16, (E, 2 * I, H), dev)
    _need(w2, "w2", torch.bfloat16, (E, H, I), dev)
    _opt(logit_bias, "logit_bias", torch.float32, (E,), dev)
    _opt(sel_bias, "sel_bias", torch.float32, (E,), dev)
    _opt(token_mask, "token_mask", torch.uint8, (T,), dev)
    if Is:
        _need(w13_s, "w13_s", torch.bfloat16, (2 * Is, H), dev)
        _need(w2_s, "w2_s", torch.bfloat16, (H, Is), dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev) if out is None else out
    _need(out, "out", torch.bfloat16, (T, H), dev)
    ws = _ws(workspace_bytes(cfg, N.MOE_STAGE_FORWARD), dev, ws)
    st = new_status(dev) if status is None else status
    b = {}
    if keep:
        b = {"logits": torch.empty(T, E, dtype=torch.float32, device=dev),
             "topk_ids": torch.empty(T, K, dtype=torch.int32, device=dev),
             "topk_w": torch.empty(T, K, dtype=torch.float32, device=dev),
             "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev)}
    ev = None
    if stage_events is not None:
        if len(stage_events) != N.MOE_NUM_STAGE_EVENTS:
            raise MoeError(f"stage_events needs {N.MOE_NUM_STAGE_EVENTS} events")
        stream = torch.cuda.current_stream(dev)
        for e in stage_events:
            if e is not None and not e.cuda_event:
                e.record(stream)  # torch creates its events lazily, on first record
        ev = (ctypes.c_void_p * N.MOE_NUM_STAGE_EVENTS)(
            *[None if e is None else e.cuda_event for e in stage_events])
    _rc(N.load().moe_forward(ctypes.byref(cfg.c()), _p(x), _p(w_router), _p(logit_bias),
                             _p(sel_bias), _p(token_mask), _p(w13), _p(w2), _p(w13_s),
                             _p(w2_s), _p(out), _p(b.get("logits")), _p(b.get("topk_ids")),
                             _p(b.get("topk_w")), _p(b.get("offsets")), _p(st), _p(ws),
                             ws.numel(), ev, _stream(dev)), "moe_forward")
    if check:
        check_status(st)
    return (out, b) if keep else out


def forward_host_workspace_bytes(cfg: Config, chunk: int) -> int:
    return int(N.load().moe_forward_host_workspace_bytes(ctypes.byref(cfg.c()), int(chunk)))


def forward_host(cfg: Config, x_host, w_router, w13, w2, logit_bias=None, sel_bias=None,
                 token_mask=None, w13_s=None, w2_s=None, out_host=None, chunk: int = 6144,
                 ws=None, status=None, check: bool = True):
    """The layer from and to host memory in one C-ABI call, transfers overlapped with the
    compute in chunks around `chunk` tokens (half-size first and last chunks, middle ones of
    at most 1.5 x chunk; see moe_forward_host). x_host / out_host are CPU bf16 tensors (pin
    them for the overlap); weights, biases and the mask are on the device."""
    dev = w13.device
    T, H, E, K, I, Is = cfg.T, cfg.H, cfg.E, cfg.K, cfg.I, cfg.I_shared
    cpu = torch.device("cpu")
    _need(x_host, "x_host", torch.bfloat16, (T, H), cpu)
    out_host = torch.empty(T, H, dtype=torch.bfloat16).pin_memory() if out_host is None \
        else out_host
    _need(out_host, "out_host", torch.bfloat16, (T, H), cpu)
    _need(w_router, "w_router", torch.bfloat16, (E, H), dev)
    _need(w13, "w13", torch.bfloat16, (E, 2 * I, H), dev)
    _need(w2, "w2", torch.bfloat16, (E, H, I), dev)
    _opt(logit_bias, "logit_bias", torch.float32, (E,), dev)
    _opt(sel_bias, "sel_bias", torch.float32, (E,), dev)
    _opt(token_mask, "token_mask", torch.uint8, (T,), dev)
    if Is:
        _need(w13_s, "w13_s", torch.bfloat16, (2 * Is, H), dev)
        _need(w2_s, "w2_s", torch.bfloat16, (H, Is), dev)
    ws = _ws(forward_host_workspace_bytes(cfg, chunk), dev, ws)
    st = new_status(dev) if status is None else status
    _rc(N.load().moe_forward_host(ctypes.byref(cfg.c()), _p(x_host), _p(w_router),
                                  _p(logit_bias), _p(sel_bias), _p(token_mask), _p(w13), _p(w2),
                                  _p(w13_s), _p(w2_s), _p(out_host), _p(st), int(chunk), _p(ws),
                                  ws.numel(), _stream(dev)), "moe_forward_host")
    if check:
        check_status(st)
    return out_host


class MoELayer:
    """A layer holding its weights and a reusable workspace sized for up to max_T tokens.

    weights: dict with w_router, w13, w2 and optionally logit_bias, sel_bias, w13_s, w2_s
    (the layout of include/moe.h)."""

    def __init__(self, cfg: Config, weights: dict, max_T: Optional[int] = None):
        self.cfg = cfg
        self.w = weights
        self.max_T = cfg.T if max_T is None else max_T
        dev = weights["w13"].device
        self.ws = _ws(workspace_bytes(cfg.with_T(self.max_T), N.MOE_STAGE_FORWARD), dev, None)
        self.status = new_status(dev)

    def forward_host(self, x_host, out_host=None, chunk: int = 6144, token_mask=None,
                     check=True):
        """The layer from pinned host memory to pinned host memory (see forward_host)."""
        T = x_host.shape[0]
        need = forward_host_workspace_bytes(self.cfg.with_T(T), chunk)
        if getattr(self, "_host_ws", None) is None or self._host_ws.numel() < need:
            self._host_ws = _ws(need, self.ws.device, None)
        w = self.w
        return forward_host(self.cfg.with_T(T), x_host, w["w_router"], w["w13"], w["w2"],
                            logit_bias=w.get("logit_bias"), sel_bias=w.get("sel_bias"),
                            token_mask=token_mask, w13_s=w.get("w13_s"), w2_s=w.get("w2_s"),
                            out_host=out_host, chunk=chunk, ws=self._host_ws,
                            status=self.status, check=check)

    def __call__(self, x, token_mask=None, out=None, keep=False, check=True, stage_events=None):
        T = x.shape[0]
        if T > self.max_T:
            raise MoeError(f"{T} tokens > the layer's max_T {self.max_T}")
        w = self.w
        return forward(self.cfg.with_T(T), x, w["w_router"], w["w13"], w["w2"],
                       logit_bias=w.get("logit_bias"), sel_bias=w.get("sel_bias"),
                       token_mask=token_mask, w13_s=w.get("w13_s"), w2_s=w.get("w2_s"),
                       out=out, ws=self.ws, status=self.status, keep=keep, check=check,
                       stage_events=stage_events)

"""CPU oracle of the top-k MoE FFN forward pass -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. The product (the CUDA library and its Python binding) never
imports, links or calls it, and the oracle imports nothing from the product.

The arithmetic lives in ``moe_oracle.c`` (plain C, built with gcc, no FMA contraction);
this module only compiles it and marshals numpy arrays. bf16 tensors travel as their
raw ``uint16`` bits.

Every function here is pinned by the CPU tests in ``tests/test_oracle_pins.py`` and
``tests/test_oracle_golden.py`` against things other than the oracle itself (closed
forms, brute force, hand-worked examples, numpy/libm in float64).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

SOFTMAX = 0
SIGMOID = 1
SQRTSOFTPLUS = 2

GCC_FLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC",
             "-std=c11", "-Wall"]


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc). Returns its path."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", *GCC_FLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_D = ctypes.c_double

_SIGS = {
    "oracle_bf16_to_f32": (_F, [ctypes.c_uint16]),
    "oracle_f32_to_bf16": (ctypes.c_uint16, [_F]),
    "oracle_f32_to_bf16_array": (None, [_P, _P, _I64]),
    "oracle_exp_rl": (_F, [_F]),
    "oracle_exp_rl_array": (None, [_P, _P, _I64]),
    "oracle_fn_array": (None, [_I, _P, _P, _I64]),
    "oracle_dot32": (_F, [_I, _P, _P]),
    "oracle_combine_bwd_fp32": (None, [_I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "oracle_router_bwd_fp32": (None, [_I, _I, _I, _P, _P, _P, _P, _I, _I, _F, _P]),
    "oracle_unpermute_fp32": (None, [_I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "oracle_sqrtsoftplus64": (_D, [_D]),
    "oracle_tree_sum32": (_F, [_P, _I]),
    "oracle_scores_fp32": (None, [_I, _P, _I, _P]),
    "oracle_select_key": (ctypes.c_uint64, [_F, _I]),
    "oracle_route_fp32": (None, [_I, _I, _I, _P, _P, _P, _I, _I, _F, _P, _P, _P]),
    "oracle_route_fp32_grouped": (None, [_I, _I, _I, _P, _P, _P, _I, _I, _F, _I, _I, _P, _P,
                                         _P]),
    "oracle_permute": (_I64, [_I, _I, _I, _P, _P, _P, _P]),
    "oracle_combine_acc_fp32": (None, [_I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "oracle_combine_fp32": (None, [_I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "oracle_logits64": (None, [_I, _I, _I, _P, _P, _P, _P]),
    "oracle_weights64": (None, [_I, _I, _I, _P, _P, _I, _I, _D, _P]),
    "oracle_expert_ffn64": (None, [_I, _I, _P, _P, _P, _P, _P]),
    "oracle_forward64": (None, [_I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P,
                                _P, _I, _P]),
    "oracle_layer_forward": (None, [_I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _P, _P,
                                    _P, _P, _I, _P, _P, _P]),
    "oracle_router_stats": (None, [_I, _I, _I, _P, _P, _P, _I, _P, _P, _P]),
    "oracle_combine_invariant": (None, [_I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "oracle_num_threads": (_I, []),
}


def lib():
    global _lib
    with _lock:
        if _lib is None:
            l = ctypes.CDLL(build())
            for name, (res, args) in _SIGS.items():
                f = getattr(l, name)
                f.restype = res
                f.argtypes = args
            _lib = l
    return _lib


# ------------------------------------------------------------------ marshalling

def _arr(a, dtype):
    """C-contiguous numpy array of the given dtype (None passes through)."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        import torch
        t = a.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            t = t.view(torch.int16)
        a = t.numpy()
    a = np.ascontiguousarray(a)
    if dtype == np.uint16 and a.dtype == np.int16:
        a = a.view(np.uint16)
    if a.dtype != dtype:
        a = a.astype(dtype)
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def bf16_to_f32(bits) -> np.ndarray:
    b = _arr(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x) -> np.ndarray:
    x = _arr(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().oracle_f32_to_bf16_array(_ptr(x), _ptr(out), x.size)
    return out


def exp_rl(x) -> np.ndarray:
    x = _arr(x, np.float32)
    out = np.empty_like(x)
    lib().oracle_exp_rl_array(_ptr(x), _ptr(out), x.size)
    return out


def _fn(which, x):
    x = _arr(x, np.float32)
    out = np.empty_like(x)
    lib().oracle_fn_array(which, _ptr(x), _ptr(out), x.size)
    return out


def ln_rl(v) -> np.ndarray:
    """The contract's fp32 natural log for v >= 1 (the sqrtsoftplus score's log1p)."""
    return _fn(0, v)


def log1p_rl(u) -> np.ndarray:
    """The contract's fp32 log1p for u >= 0 (Goldberg's formula over ln_rl)."""
    return _fn(1, u)


def sqrtsoftplus_rl(x) -> np.ndarray:
    """The contract's fp32 sqrtsoftplus score."""
    return _fn(2, x)


def sqrtsoftplus64(x) -> np.ndarray:
    """sqrt(softplus(x)) in double with libm."""
    f = lib().oracle_sqrtsoftplus64
    return np.array([f(float(v)) for v in np.ravel(x)], np.float64).reshape(np.shape(x))


def tree_sum32(v) -> np.float32:
    v = _arr(v, np.float32)
    return np.float32(lib().oracle_tree_sum32(_ptr(v), v.size))


def scores_fp32(logits_row, score_fn: int) -> np.ndarray:
    l = _arr(logits_row, np.float32)
    s = np.empty_like(l)
    lib().oracle_scores_fp32(l.size, _ptr(l), score_fn, _ptr(s))
    return s


def select_key(c: float, idx: int) -> int:
    return int(lib().oracle_select_key(float(np.float32(c)), idx))


def route_fp32(logits, K: int, score_fn: int, renorm: bool, route_scale: float = 1.0,
               sel_bias=None, mask=None, n_group: int = 0, topk_group: int = 0):
    """FP32-contract routing (group-limited when n_group > 1). Returns (ids [T,K] int32,
    w [T,K] fp32, status [2] int64)."""
    l = _arr(logits, np.float32)
    T, E = l.shape
    sb = _arr(sel_bias, np.float32)
    m = _arr(mask, np.uint8)
    ids = np.empty((T, K), np.int32)
    w = np.empty((T, K), np.float32)
    st = np.zeros(2, np.int64)
    lib().oracle_route_fp32_grouped(T, E, K, _ptr(l), _ptr(sb), _ptr(m), score_fn,
                                    int(bool(renorm)), float(route_scale), int(n_group),
                                    int(topk_group), _ptr(ids), _ptr(w), _ptr(st))
    return ids, w, st


def permute(ids, E: int):
    """Counting sort of the assignments. Returns (offsets, perm_token, dest_row, n_bad)."""
    ids = _arr(ids, np.int32)
    T, K = ids.shape
    offsets = np.empty(E + 1, np.int32)
    perm_token = np.full(T * K, -1, np.int32)
    dest_row = np.empty(T * K, np.int32)
    bad = lib().oracle_permute(T, K, E, _ptr(ids), _ptr(offsets), _ptr(perm_token),
                               _ptr(dest_row))
    return offsets, perm_token, dest_row.reshape(T, K), int(bad)


def combine_acc_fp32(y, w, dest_row, y_shared=None, mask=None) -> np.ndarray:
    y = _arr(y, np.uint16)
    w = _arr(w, np.float32)
    d = _arr(dest_row, np.int32)
    T, K = w.shape
    H = y.shape[-1]
    ys = _arr(y_shared, np.uint16)
    m = _arr(mask, np.uint8)
    acc = np.empty((T, H), np.float32)
    lib().oracle_combine_acc_fp32(T, K, H, _ptr(y), _ptr(w), _ptr(d), _ptr(ys), _ptr(m),
                                  _ptr(acc))
    return acc


def combine_fp32(y, w, dest_row, y_shared=None, mask=None) -> np.ndarray:
    """FP32-contract weighted combine; returns bf16 bits [T,H] as uint16."""
    y = _arr(y, np.uint16)
    w = _arr(w, np.float32)
    d = _arr(dest_row, np.int32)
    T, K = w.shape
    H = y.shape[-1]
    ys = _arr(y_shared, np.uint16)
    m = _arr(mask, np.uint8)
    out = np.empty((T, H), np.uint16)
    lib().oracle_combine_fp32(T, K, H, _ptr(y), _ptr(w), _ptr(d), _ptr(ys), _ptr(m),
                              _ptr(out))
    return out


def combine_invariant(y, w, dest_row, y_shared=None, mask=None) -> np.ndarray:
    """Order-invariant combine (canonical-order double sum of exact products); bf16 bits."""
    y = _arr(y, np.uint16)
    w = _arr(w, np.float32)
    d = _arr(dest_row, np.int32)
    T, K = w.shape
    H = y.shape[-1]
    ys = _arr(y_shared, np.uint16)
    m = _arr(mask, np.uint8)
    out = np.empty((T, H), np.uint16)
    lib().oracle_combine_invariant(T, K, H, _ptr(y), _ptr(w), _ptr(d), _ptr(ys), _ptr(m),
                                   _ptr(out))
    return out


def logits64(x, w_router, logit_bias=None) -> np.ndarray:
    x = _arr(x, np.uint16)
    wr = _arr(w_router, np.uint16)
    lb = _arr(logit_bias, np.float32)
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), np.float64)
    lib().oracle_logits64(T, H, E, _ptr(x), _ptr(wr), _ptr(lb), _ptr(out))
    return out


def weights64(logits, ids, score_fn: int, renorm: bool, route_scale: float = 1.0):
    l = _arr(logits, np.float64)
    ids = _arr(ids, np.int32)
    T, E = l.shape
    K = ids.shape[1]
    w = np.empty((T, K), np.float64)
    lib().oracle_weights64(T, E, K, _ptr(l), _ptr(ids), score_fn, int(bool(renorm)),
                           float(route_scale), _ptr(w))
    return w


def expert_ffn64(x_row, w13_e, w2_e, return_h: bool = False):
    x = _arr(x_row, np.uint16).reshape(-1)
    w13 = _arr(w13_e, np.uint16)
    w2 = _arr(w2_e, np.uint16)
    H = x.size
    I = w13.shape[0] // 2
    y = np.empty(H, np.float64)
    h = np.empty(I, np.float64) if return_h else None
    lib().oracle_expert_ffn64(H, I, _ptr(x), _ptr(w13), _ptr(w2), _ptr(y), _ptr(h))
    return (y, h) if return_h else y


def forward64(x, ids, w64, w13, w2, w13_s=None, w2_s=None, mask=None, sel=None):
    """Layer output in double for given routes; rows `sel` only (all when None)."""
    x = _arr(x, np.uint16)
    ids = _arr(ids, np.int32)
    w64 = _arr(w64, np.float64)
    w13 = _arr(w13, np.uint16)
    w2 = _arr(w2, np.uint16)
    w13s = _arr(w13_s, np.uint16)
    w2s = _arr(w2_s, np.uint16)
    m = _arr(mask, np.uint8)
    T, H = x.shape
    K = ids.shape[1]
    E = w13.shape[0]
    I = w13.shape[1] // 2
    Is = 0 if w13s is None else w13s.shape[0] // 2
    s = None if sel is None else _arr(sel, np.int32)
    n = T if s is None else s.size
    out = np.empty((n, H), np.float64)
    lib().oracle_forward64(T, H, E, K, I, Is, _ptr(x), _ptr(ids), _ptr(w64), _ptr(m),
                           _ptr(w13), _ptr(w2), _ptr(w13s), _ptr(w2s), _ptr(s), n, _ptr(out))
    return out


def layer_forward(shape, tensors, sel):
    """Whole layer on the CPU for the tokens in `sel` (the timed CPU baseline).

    Returns (ids [n,K], out [n,H] double)."""
    x = _arr(tensors["x"], np.uint16)
    wr = _arr(tensors["w_router"], np.uint16)
    lb = _arr(tensors.get("logit_bias"), np.float32)
    sb = _arr(tensors.get("sel_bias"), np.float32)
    w13 = _arr(tensors["w13"], np.uint16)
    w2 = _arr(tensors["w2"], np.uint16)
    w13s = _arr(tensors.get("w13_s"), np.uint16)
    w2s = _arr(tensors.get("w2_s"), np.uint16)
    s = _arr(sel, np.int32)
    n = s.size
    ids = np.empty((n, shape.K), np.int32)
    out = np.empty((n, shape.H), np.float64)
    lib().oracle_layer_forward(shape.H, shape.E, shape.K, shape.I,
                               shape.I_shared if w13s is not None else 0, shape.score_fn,
                               int(shape.renorm), float(shape.route_scale), _ptr(x), _ptr(wr),
                               _ptr(lb), _ptr(sb), _ptr(w13), _ptr(w2), _ptr(w13s), _ptr(w2s),
                               n, _ptr(s), _ptr(ids), _ptr(out))
    return ids, out


def router_stats(logits, ids, score_fn: int, mask=None):
    """(counts [E] int64, mean_prob [E] float64, aux float) of one routed batch."""
    l = _arr(logits, np.float32)
    ids = _arr(ids, np.int32)
    m = _arr(mask, np.uint8)
    T, E = l.shape
    K = ids.shape[1]
    counts = np.empty(E, np.int64)
    mp = np.empty(E, np.float64)
    aux = np.zeros(1, np.float64)
    lib().oracle_router_stats(T, E, K, _ptr(l), _ptr(ids), _ptr(m), score_fn, _ptr(counts),
                              _ptr(mp), _ptr(aux))
    return counts, mp, float(aux[0])


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# ------------------------------------------------------------------ backward (FP32 contract)

def dot32(a, b) -> np.float32:
    """The contract's fp32 dot product of two bf16 rows (8-element chunks over 32 lanes)."""
    a = _arr(a, np.uint16).reshape(-1)
    b = _arr(b, np.uint16).reshape(-1)
    return np.float32(lib().oracle_dot32(a.size, _ptr(a), _ptr(b)))


def combine_bwd_fp32(dout, y, w, dest_row, rows, mask=None, shared=False):
    """(dw [T,K] fp32, dy [rows,H] bf16 bits, dy_shared [T,H] bf16 bits or None)."""
    g = _arr(dout, np.uint16)
    yy = _arr(y, np.uint16)
    ww = _arr(w, np.float32)
    d = _arr(dest_row, np.int32)
    m = _arr(mask, np.uint8)
    T, H = g.shape
    K = d.shape[1]
    dw = np.empty((T, K), np.float32)
    dy = np.zeros((max(rows, 1), H), np.uint16)
    dys = np.empty((T, H), np.uint16) if shared else None
    lib().oracle_combine_bwd_fp32(T, K, H, _ptr(g), _ptr(yy), _ptr(ww), _ptr(d), _ptr(m),
                                  _ptr(dw), _ptr(dy), _ptr(dys))
    return dw, dy[:rows], dys


def router_bwd_fp32(logits, ids, dw, score_fn: int, renorm: bool, route_scale: float = 1.0,
                    mask=None):
    """dlogits [T,E] fp32 of the contract's router backward."""
    l = _arr(logits, np.float32)
    i = _arr(ids, np.int32)
    g = _arr(dw, np.float32)
    m = _arr(mask, np.uint8)
    T, E = l.shape
    K = i.shape[1]
    out = np.empty((T, E), np.float32)
    lib().oracle_router_bwd_fp32(T, E, K, _ptr(l), _ptr(i), _ptr(g), _ptr(m), score_fn,
                                 int(bool(renorm)), float(route_scale), _ptr(out))
    return out


def unpermute_fp32(dx_rows, dest_row, dx_shared=None, dx_router=None, mask=None):
    """dx [T,H] bf16 bits: the rank-order sum of a token's row gradients, then the shared
    expert's and the router's terms, rounded once."""
    r = _arr(dx_rows, np.uint16)
    d = _arr(dest_row, np.int32)
    s = _arr(dx_shared, np.uint16)
    q = _arr(dx_router, np.uint16)
    m = _arr(mask, np.uint8)
    T, K = d.shape
    H = r.shape[1]
    out = np.empty((T, H), np.uint16)
    lib().oracle_unpermute_fp32(T, K, H, _ptr(r), _ptr(d), _ptr(s), _ptr(q), _ptr(m),
                                _ptr(out))
    return out

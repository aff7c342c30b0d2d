"""moe_permute_noalloc: the dispatch entry point for callers that cannot allocate device
memory (it keeps its scratch in a fixed array inside the library instead of taking a
workspace). Checked through the C ABI against moe_permute and against the oracle's
counting sort, on two calls in a row with different inputs so that anything left in the
shared scratch by the first call would show up in the second. (Its size limit is checked
on the host, in test_abi_cpu.py.) This file sorts last so that a run stopping at its
first failure has run every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from deterministic_invariant_routing_b200 import _native as N
from deterministic_invariant_routing_b200 import moe, synthetic

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _ids(T, K, E, seed):
    rng = np.random.default_rng(seed)
    p = rng.dirichlet(np.full(E, 0.3))
    ids = np.stack([rng.choice(E, K, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    ids[rng.random(T) < 0.1] = -1
    return torch.from_numpy(ids).to(DEV)


def _noalloc(cfg, ids, x):
    T, K, E, H = cfg.T, cfg.K, cfg.E, cfg.H
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm_token = torch.full((T * K,), -1, dtype=torch.int32, device=DEV)
    dest_row = torch.empty(T, K, dtype=torch.int32, device=DEV)
    x_perm = torch.empty(T * K, H, dtype=torch.bfloat16, device=DEV)
    status = moe.new_status(DEV)
    rc = N.load().moe_permute_noalloc(ctypes.byref(cfg.c()), _p(ids), _p(x), _p(offsets),
                                      _p(perm_token), _p(dest_row), _p(x_perm), _p(status),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == N.MOE_OK, N.status_string(rc)
    torch.cuda.synchronize()
    return offsets, perm_token, dest_row, x_perm, status


def test_permute_noalloc_matches_permute_and_oracle_on_two_calls():
    for call, (T, K, E, H) in enumerate([(3001, 8, 128, 256), (777, 6, 256, 128)]):
        cfg = moe.Config(T=T, H=H, E=E, K=K, I=128)
        ids = _ids(T, K, E, seed=call)
        x = synthetic.normal_bf16(T, H, 1.0, 11 + call, "x", device=DEV)
        r_off, r_perm, r_dest, r_xp = moe.permute(cfg, ids, x=x)
        offsets, perm_token, dest_row, x_perm, status = _noalloc(cfg, ids, x)
        n = int(r_off[-1])
        # against the workspace entry point
        assert torch.equal(offsets, r_off)
        assert torch.equal(perm_token[:n], r_perm[:n])
        assert torch.equal(dest_row, r_dest)
        assert torch.equal(x_perm[:n].view(torch.int16), r_xp[:n].view(torch.int16))
        assert int(status.abs().sum()) == 0
        # against the oracle's stable counting sort, bit for bit
        o_off, o_perm, o_dest, _ = oracle.permute(ids.cpu().numpy(), E)
        assert np.array_equal(offsets.cpu().numpy(), o_off)
        assert int(o_off[-1]) == n
        assert np.array_equal(perm_token[:n].cpu().numpy(), o_perm[:n])
        assert np.array_equal(dest_row.cpu().numpy().reshape(-1), o_dest.reshape(-1))
        xb = x.cpu().view(torch.int16).numpy()
        assert np.array_equal(x_perm[:n].cpu().view(torch.int16).numpy(), xb[o_perm[:n]])

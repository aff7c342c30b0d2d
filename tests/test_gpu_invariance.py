"""Level-3 parity: GPU results are bitwise batch-invariant.

The same target tokens are run alone, in slices of every batch size, among fillers at
random positions, behind random left/right padding (with the padding masked, and with
no mask so the pad rows are processed like tokens), in a random token order, and as
prefill chunks of 256/512/2048 tokens in separate calls. Every variant must give the
same bits for the targets' logits, expert ids, weights and layer output
("DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 1 and the DSV4-WS1-1
bucket: routing / dispatch / combine align across batch and padding sweeps).
"""
import numpy as np
import pytest
import torch

from deterministic_invariant_routing_b200 import moe, synthetic
from helpers import DEV, REPORT, bits, near_tie_count

pytestmark = pytest.mark.gpu


class Sweep:
    def __init__(self, name, n_targets, max_T):
        self.s = synthetic.shape(name, T=max_T)
        self.w = synthetic.make_weights(self.s, device=DEV)
        self.cfg = moe.Config.of(self.s)
        self.layer = moe.MoELayer(self.cfg, self.w, max_T=max_T)
        self.targets = synthetic.make_tokens(self.s, n_targets, seed=5, device=DEV)
        self.n = n_targets
        self.fill_seed = 1000

    def fillers(self, n):
        self.fill_seed += 1
        return synthetic.make_tokens(self.s, n, seed=self.fill_seed, device=DEV, tag="fill")

    def run(self, x, mask=None):
        out, b = self.layer(x, token_mask=mask, keep=True)
        return {"out": out, "logits": b["logits"], "ids": b["topk_ids"], "w": b["topk_w"]}

    def pick(self, r, rows):
        idx = torch.as_tensor(rows, dtype=torch.long, device=DEV)
        return {k: v.index_select(0, idx) for k, v in r.items()}


def same(a, b, what):
    for k in ("logits", "ids", "w", "out"):
        assert np.array_equal(bits(a[k]), bits(b[k])), f"{what}: {k} differs"


def concat(parts):
    return {k: torch.cat([p[k] for p in parts]) for k in parts[0]}


BATCHES = [1, 2, 3, 7, 16, 64, 255, 256, 1000, 2047, 2048, 2049, 4096, 8192, 16384]


@pytest.fixture(scope="module")
def sweep():
    return Sweep("qwen3_30b_a3b", 2048, 16384 + 512)


def test_batch_size_sweep(sweep):
    ref = sweep.run(sweep.targets)
    rng = np.random.default_rng(0)
    for B in BATCHES:
        if B <= sweep.n:
            parts = [sweep.run(sweep.targets[i:i + B]) for i in range(0, sweep.n, B)]
            got = concat(parts)
        else:
            pos = np.sort(rng.choice(B, sweep.n, replace=False))
            x = sweep.fillers(B)
            x[torch.as_tensor(pos, device=DEV)] = sweep.targets
            got = sweep.pick(sweep.run(x), pos)
        same(got, ref, f"batch {B}")
    lg = ref["logits"].cpu().numpy()
    REPORT.append(f"level 3 batch sweep {BATCHES[0]}..{BATCHES[-1]}: {sweep.n} target tokens "
                  f"bit-identical in {len(BATCHES)} batch sizes; near ties among them (K-th vs "
                  f"K+1-th choice within 1 ulp): {near_tie_count(lg, sweep.s)}")


@pytest.mark.parametrize("masked", [True, False])
def test_left_right_padding(sweep, masked):
    ref = sweep.run(sweep.targets)
    rng = np.random.default_rng(1 + masked)
    for _ in range(4):
        left, right = (int(v) for v in rng.integers(0, 300, 2))
        T = left + sweep.n + right
        x = torch.zeros(T, sweep.s.H, dtype=torch.bfloat16, device=DEV)
        x[:left] = sweep.fillers(left) if left else x[:0]
        x[left + sweep.n:] = sweep.fillers(right) if right else x[:0]
        x[left:left + sweep.n] = sweep.targets
        mask = None
        if masked:
            mask = torch.zeros(T, dtype=torch.uint8, device=DEV)
            mask[left:left + sweep.n] = 1
        r = sweep.run(x, mask)
        got = sweep.pick(r, np.arange(left, left + sweep.n))
        same(got, ref, f"padding {left}/{right} masked={masked}")
        if masked:
            assert np.all(bits(r["out"][:left]) == 0) and np.all(bits(r["out"][left + sweep.n:]) == 0)
            assert torch.all(r["ids"][:left] == -1)


def test_token_permutation(sweep):
    ref = sweep.run(sweep.targets)
    for seed in range(3):
        perm = synthetic.random_permutation(sweep.n, seed).to(DEV)
        r = sweep.run(sweep.targets[perm])
        inv = torch.empty_like(perm)
        inv[perm] = torch.arange(sweep.n, device=DEV)
        got = {k: v.index_select(0, inv) for k, v in r.items()}
        same(got, ref, f"permutation {seed}")


@pytest.mark.parametrize("chunk", [256, 512, 2048])
def test_prefill_chunks(sweep, chunk):
    ref = sweep.run(sweep.targets)
    got = concat([sweep.run(sweep.targets[i:i + chunk]) for i in range(0, sweep.n, chunk)])
    same(got, ref, f"chunks of {chunk}")


def test_sigmoid_shared_expert_layer_invariance():
    """The DeepSeek-style layer (sigmoid router, selection bias, route_scale, shared
    expert) under the same kinds of variation, on fewer targets."""
    sw = Sweep("dsv_sigmoid", 512, 4096 + 64)
    ref = sw.run(sw.targets)
    same(concat([sw.run(sw.targets[i:i + 7]) for i in range(0, sw.n, 7)]), ref, "slices of 7")
    rng = np.random.default_rng(3)
    pos = np.sort(rng.choice(4096, sw.n, replace=False))
    x = sw.fillers(4096)
    x[torch.as_tensor(pos, device=DEV)] = sw.targets
    same(sw.pick(sw.run(x), pos), ref, "among fillers")
    perm = synthetic.random_permutation(sw.n, 9).to(DEV)
    r = sw.run(sw.targets[perm])
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(sw.n, device=DEV)
    same({k: v.index_select(0, inv) for k, v in r.items()}, ref, "permutation")
    T = sw.n + 40
    x = torch.zeros(T, sw.s.H, dtype=torch.bfloat16, device=DEV)
    x[17:17 + sw.n] = sw.targets
    mask = torch.zeros(T, dtype=torch.uint8, device=DEV)
    mask[17:17 + sw.n] = 1
    same(sw.pick(sw.run(x, mask), np.arange(17, 17 + sw.n)), ref, "masked padding")


@pytest.mark.parametrize("name,T,chunks", [("qwen3_30b_a3b", 4096, (1000, 2048, 4096, 8192)),
                                           ("tiny", 333, (7, 64, 333)),
                                           ("dsv_sigmoid", 1500, (512,))])
def test_forward_host_chunked_equals_forward(name, T, chunks):
    """The host-memory entry point (chunked, copies overlapped) gives the bits of one
    moe_forward on device memory, for any chunk size, with and without a mask."""
    s, d = synthetic.make_layer(name, T=T, device=DEV)
    cfg = moe.Config.of(s)
    mask = synthetic.random_mask(T, 0.85, 3).to(DEV)
    w = dict(logit_bias=d["logit_bias"], sel_bias=d["sel_bias"], w13_s=d["w13_s"], w2_s=d["w2_s"])
    x_host = d["x"].cpu().pin_memory()
    for m in (None, mask):
        ref = moe.forward(cfg, d["x"], d["w_router"], d["w13"], d["w2"], token_mask=m, **w)
        for c in chunks:
            out = moe.forward_host(cfg, x_host, d["w_router"], d["w13"], d["w2"], token_mask=m,
                                   chunk=c, **w)
            assert np.array_equal(bits(out), bits(ref)), (name, c, m is not None)

"""The layer forward captured in a CUDA graph. The entry points only enqueue work on the
caller's stream (no host synchronisation, no allocation), so a capture of moe_forward
replays to the eager call's bits, and new tokens copied into the captured input buffer
are routed and computed like an eager call on them."""
import numpy as np
import pytest
import torch

from deterministic_invariant_routing_b200 import moe, synthetic
from deterministic_invariant_routing_b200 import _native as N
from helpers import DEV, REPORT, bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,T", [("tiny", 64), ("qwen3_30b_a3b", 1), ("qwen3_30b_a3b", 256),
                                    ("qwen3_30b_a3b", 4096), ("dsv_sigmoid", 128)])
def test_forward_replayed_from_cuda_graph(name, T):
    s, d = synthetic.make_layer(name, T=T, device=DEV)
    cfg = moe.Config.of(s)
    w = dict(w_router=d["w_router"], w13=d["w13"], w2=d["w2"], logit_bias=d["logit_bias"],
             sel_bias=d["sel_bias"], w13_s=d["w13_s"], w2_s=d["w2_s"])
    ref = moe.forward(cfg, d["x"], **w)
    x_buf = d["x"].clone()
    out = torch.empty_like(ref)
    ws = torch.empty(moe.workspace_bytes(cfg, N.MOE_STAGE_FORWARD), dtype=torch.uint8,
                     device=DEV)
    st = moe.new_status(DEV)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # an uncaptured call on the capture stream first
        moe.forward(cfg, x_buf, out=out, ws=ws, status=st, check=False, **w)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.forward(cfg, x_buf, out=out, ws=ws, status=st, check=False, **w)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), bits(ref))
    moe.check_status(st)
    x2 = synthetic.make_tokens(s, T, seed=s.seed + 99, device=DEV)
    ref2 = moe.forward(cfg, x2, **w)
    x_buf.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), bits(ref2))
    moe.check_status(st)
    # latency of one call, eager against replay (reported, not asserted)
    def per_call_us(fn, n=20):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n * 1e3
    eager = per_call_us(lambda: moe.forward(cfg, x_buf, out=out, ws=ws, status=st, check=False,
                                            **w))
    replay = per_call_us(g.replay)
    REPORT.append(f"cuda graph {name} T={T}: replay bit-equal to eager; {eager:.1f} us per "
                  f"eager call, {replay:.1f} us per replay")

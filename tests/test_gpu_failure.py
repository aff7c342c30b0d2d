"""Fail-closed detection on the GPU without a fault ("DSV4 Flash MoE Train-Inference
Consistency Roadmap", Follow-Up Issue Buckets: a mismatch fails closed). The pipelines'
bounded wait is made to run out on a barrier that nothing arrives on: the kernel returns,
the device status counts a pipeline timeout, the binding raises, and the context stays
usable for the next call."""
import pytest
import torch

from deterministic_invariant_routing_b200 import _native as N
from deterministic_invariant_routing_b200 import moe, synthetic
from helpers import DEV, bits

pytestmark = pytest.mark.gpu


def test_pipeline_wait_gives_up_and_is_reported():
    st = moe.pipeline_wait_selftest(DEV, limit_cycles=200_000, check=False)
    torch.cuda.synchronize()
    words = st.cpu().tolist()
    assert words[N.MOE_ST_PIPE_TIMEOUT] == 1 and sum(words) == 1
    with pytest.raises(moe.StatusError, match="pipeline_timeout"):
        moe.pipeline_wait_selftest(DEV, limit_cycles=200_000)


def test_context_usable_after_a_timeout():
    moe.pipeline_wait_selftest(DEV, limit_cycles=200_000, check=False)
    s, d = synthetic.make_layer("tiny", device=DEV)
    cfg = moe.Config.of(s)
    a = moe.forward(cfg, d["x"], d["w_router"], d["w13"], d["w2"])
    b = moe.forward(cfg, d["x"], d["w_router"], d["w13"], d["w2"])
    torch.cuda.synchronize()
    assert (bits(a) == bits(b)).all()

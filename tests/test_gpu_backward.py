"""The layer's backward (moe_backward) on the GPU against the oracle.

* level 1 (bit-exact): the routing-weight gradient d_topk_w = dot32(dout, y) given the
  GPU's expert outputs y, and dlogits from the GPU's logits and d_topk_w (the FP32
  contract's router backward);
* level 2 (tolerance): dx, the expert weight gradients, the router weight gradient and
  the shared expert's gradients against the FP64 backward on the same logits and routes:
  dx per token row, every weight gradient element by element within twice a first-order
  error bound of its computation and within a root-sum-square allowance that a misplaced
  element exceeds (both derived in helpers.py), and per matrix in Frobenius norm; at T = 4096 the checked experts include the most and the least loaded
  (several 64-row k-blocks each) and the router's product runs in 16 token chunks;
* determinism and batch invariance: two calls give the same bits; a token's dx does not
  depend on the other tokens of the batch; experts without rows get exact zeros.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward64 as B
from deterministic_invariant_routing_b200 import moe, synthetic
from helpers import (DEV, REPORT, WGRAD_EXPERT_CQ, WGRAD_ROUTER_CQ, assert_within_bounds, bits,
                     layer, wgrad_bounds64)

pytestmark = pytest.mark.gpu

DX_ROW_REL = 2e-2     # dx: per token row, max |gpu - ref| / max |ref|
DW_FRO_REL = 1e-2     # weight gradients: ||gpu - ref||_F / ||ref||_F per matrix


class LazyF64:
    """Expert weights as float64, one expert at a time (keeps host memory small)."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return B.bf16_to_f64(bits(self.t[int(e)].cpu()))


def run(name, T, keep=None, seed=0, **over):
    s, d, cfg = layer(name, T, **over)
    mask = None if keep is None else synthetic.random_mask(T, keep, 31 + seed).to(DEV)
    out, b = moe.forward(cfg, d["x"], d["w_router"], d["w13"], d["w2"],
                         logit_bias=d["logit_bias"], sel_bias=d["sel_bias"], token_mask=mask,
                         w13_s=d["w13_s"], w2_s=d["w2_s"], keep=True)
    dout = synthetic.normal_bf16(T, s.H, 1.0, s.seed + 77 + seed, "fill").to(DEV)
    g = moe.backward(cfg, d["x"], d["w_router"], d["w13"], d["w2"], b["logits"], b["topk_ids"],
                     b["topk_w"], dout, token_mask=mask, w13_s=d["w13_s"], w2_s=d["w2_s"],
                     keep=True)
    torch.cuda.synchronize()
    return s, d, cfg, mask, b, dout, g


def fro_rel(gpu, ref):
    g = np.asarray(gpu, np.float64)
    den = np.linalg.norm(ref)
    return np.linalg.norm(g - ref) / den if den > 0 else np.linalg.norm(g)


def check_backward(name, T, keep=None, **over):
    s, d, cfg, mask, b, dout, g = run(name, T, keep, **over)
    mask_np = None if mask is None else mask.cpu().numpy()
    ids = b["topk_ids"].cpu().numpy()
    lg = b["logits"].cpu().numpy()

    # level 1: d_topk_w from the GPU's own y (the stage API runs the same kernels)
    offsets, perm_token, dest_row, x_perm = moe.permute(cfg, b["topk_ids"], x=d["x"])
    y, _ = moe.grouped_ffn(cfg, d["x"], x_perm, perm_token, offsets, d["w13"], d["w2"],
                           d["w13_s"], d["w2_s"])
    torch.cuda.synchronize()
    rows = int(offsets[-1].item())
    r_dw, _, _ = oracle.combine_bwd_fp32(bits(dout.cpu()), bits(y.cpu()), b["topk_w"].cpu().numpy(),
                                         dest_row.cpu().numpy(), rows, mask=mask_np)
    assert np.array_equal(bits(g["d_topk_w"].cpu()), r_dw.view(np.uint32))
    # level 1: dlogits from the GPU's logits and d_topk_w
    r_dl = oracle.router_bwd_fp32(lg, ids, g["d_topk_w"].cpu().numpy(), s.score_fn, s.renorm,
                                  s.route_scale, mask=mask_np)
    assert np.array_equal(bits(g["dlogits"].cpu()), r_dl.view(np.uint32))

    # level 2: everything against the FP64 backward on the same logits and routes (the
    # forward's logits are checked against FP64 by the layer tests)
    x64 = B.bf16_to_f64(bits(d["x"].cpu()))
    wr64 = B.bf16_to_f64(bits(d["w_router"].cpu()))
    used = np.unique(ids[ids >= 0])
    load = np.bincount(ids[ids >= 0], minlength=s.E)
    check_e = set(int(e) for e in used[:: max(1, used.size // 6)])
    check_e |= {int(used[np.argmax(load[used])]), int(used[np.argmin(load[used])])}
    w13_s64 = None if d["w13_s"] is None else B.bf16_to_f64(bits(d["w13_s"].cpu()))
    w2_s64 = None if d["w2_s"] is None else B.bf16_to_f64(bits(d["w2_s"].cpu()))
    dout64 = B.bf16_to_f64(bits(dout.cpu()))
    l64 = lg.astype(np.float64)
    ref = B.layer_backward64(dout64, x64, wr64, LazyF64(d["w13"]), LazyF64(d["w2"]), ids,
                             s.score_fn, s.renorm, s.route_scale, mask=mask_np, w13_s=w13_s64,
                             w2_s=w2_s64, logits=l64, experts=check_e)
    sc = wgrad_bounds64(dout64, x64, l64, LazyF64(d["w13"]), LazyF64(d["w2"]), ids, s.score_fn,
                        s.renorm, s.route_scale, mask=mask_np, w13_s=w13_s64, w2_s=w2_s64,
                        experts=check_e)
    gdx = g["dx"].float().cpu().numpy().astype(np.float64)
    den = np.maximum(np.abs(ref["dx"]).max(axis=1), 1e-30)
    live = np.abs(ref["dx"]).max(axis=1) > 0
    rel = np.abs(gdx - ref["dx"]).max(axis=1) / den
    assert np.all(rel[live] <= DX_ROW_REL), rel.max()
    if mask_np is not None:
        assert np.all(bits(g["dx"].cpu())[mask_np == 0] == 0)
    worst = {}
    got = {"dw_router": g["dw_router"].cpu().numpy()}
    want = {"dw_router": ref["dwr"]}
    for e in sorted(check_e):
        got[f"dw13[{e}]"], want[f"dw13[{e}]"] = g["dw13"][e].cpu().numpy(), ref["dw13"][e]
        got[f"dw2[{e}]"], want[f"dw2[{e}]"] = g["dw2"][e].cpu().numpy(), ref["dw2"][e]
    if s.I_shared:
        got["dw13_s"], want["dw13_s"] = g["dw13_s"].cpu().numpy(), ref["dw13_s"]
        got["dw2_s"], want["dw2_s"] = g["dw2_s"].cpu().numpy(), ref["dw2_s"]
    for k in got:
        cq = WGRAD_ROUTER_CQ if k == "dw_router" else WGRAD_EXPERT_CQ
        worst[k] = assert_within_bounds(got[k], want[k], sc[k], cq, k)
        assert fro_rel(got[k], want[k]) <= DW_FRO_REL, k
    REPORT.append(f"backward {name} T={T}: dx max row rel err {rel[live].max():.3e}; weight "
                  f"gradients use at most {max(worst.values()):.3f} of their element-wise "
                  f"bounds (experts {sorted(check_e)}, rows {load[sorted(check_e)].tolist()})")
    # experts with no rows: exact zeros
    unused = np.setdiff1d(np.arange(s.E), used)
    for e in unused[:4]:
        assert not g["dw13"][e].any() and not g["dw2"][e].any()
    return s, d, cfg, mask, b, dout, g


def test_backward_tiny():
    check_backward("tiny", 64)


def test_backward_tiny_masked():
    check_backward("tiny", 64, keep=0.6)


def test_backward_qwen3_30b_a3b_shape():
    check_backward("qwen3_30b_a3b", 96, keep=0.8)


def test_backward_qwen3_30b_a3b_long_k():
    """T = 4096 on the 30B-A3B layer: experts own hundreds to thousands of rows (many
    64-row k-blocks, tiles dealt by K length), and the router's weight gradient runs in
    16 chunks of 256 tokens summed in order -- the weight-gradient path at full depth."""
    check_backward("qwen3_30b_a3b", 4096, keep=0.9)


def test_backward_dspark_top1_no_renorm():
    check_backward("dspark", 48)


def test_backward_dsv_sigmoid_shared():
    check_backward("dsv_sigmoid", 40)


def test_backward_dsv_sqrtsoftplus_grouped():
    check_backward("dsv_sigmoid", 32, score_fn=synthetic.SQRTSOFTPLUS, n_group=8, topk_group=4)


def test_backward_repeatable_and_batch_invariant_dx():
    """Two calls: identical bits everywhere. A token's dx is the same in a batch of 777 and
    in the batch of its first 300 tokens (weight gradients are sums over the batch and
    legitimately differ)."""
    s, d, cfg, mask, b, dout, g1 = run("qwen3_30b_a3b", 777)
    g2 = moe.backward(cfg, d["x"], d["w_router"], d["w13"], d["w2"], b["logits"], b["topk_ids"],
                      b["topk_w"], dout, keep=True)
    torch.cuda.synchronize()
    for k in g1:
        if g1[k] is not None:
            assert torch.equal(g1[k].view(torch.int8) if g1[k].dtype != torch.bfloat16 else
                               g1[k].view(torch.int16),
                               g2[k].view(torch.int8) if g2[k].dtype != torch.bfloat16 else
                               g2[k].view(torch.int16)), k
    n = 300
    c2 = cfg.with_T(n)
    g3 = moe.backward(c2, d["x"][:n].contiguous(), d["w_router"], d["w13"], d["w2"],
                      b["logits"][:n].contiguous(), b["topk_ids"][:n].contiguous(),
                      b["topk_w"][:n].contiguous(), dout[:n].contiguous(), keep=True)
    torch.cuda.synchronize()
    assert np.array_equal(bits(g3["dx"].cpu()), bits(g1["dx"][:n].cpu()))
    assert np.array_equal(bits(g3["dlogits"].cpu()), bits(g1["dlogits"][:n].cpu()))
    # the weight gradient of the sub-batch is close to, not equal to, the full one
    assert not torch.equal(g3["dw_router"], g1["dw_router"])


def test_backward_zero_tokens_gives_zero_weight_gradients():
    s, d, cfg = layer("tiny", 64)
    c0 = cfg.with_T(0)
    e = torch.empty
    g = moe.backward(c0, e(0, s.H, dtype=torch.bfloat16, device=DEV), d["w_router"], d["w13"],
                     d["w2"], e(0, s.E, device=DEV), e(0, s.K, dtype=torch.int32, device=DEV),
                     e(0, s.K, device=DEV), e(0, s.H, dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert not g["dw13"].any() and not g["dw2"].any() and not g["dw_router"].any()


@pytest.mark.parametrize("name,T,keep", [("qwen3_30b_a3b", 300, 0.8), ("dsv_sigmoid", 64, None)])
def test_forward_train_and_saved_backward_equal_the_plain_calls(name, T, keep):
    """moe_forward_train gives moe_forward's bits and leaves the intermediates; the backward
    reusing them gives the recomputing backward's bits, for every output."""
    s, d, cfg = layer(name, T)
    mask = None if keep is None else synthetic.random_mask(T, keep, 5).to(DEV)
    kw = dict(logit_bias=d["logit_bias"], sel_bias=d["sel_bias"], token_mask=mask,
              w13_s=d["w13_s"], w2_s=d["w2_s"])
    out, b = moe.forward(cfg, d["x"], d["w_router"], d["w13"], d["w2"], keep=True, **kw)
    ws = moe.backward_workspace(cfg, DEV)
    out_t, bt = moe.forward_train(cfg, d["x"], d["w_router"], d["w13"], d["w2"], ws, **kw)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out_t.cpu()), bits(out.cpu()))
    for k in ("logits", "topk_ids", "topk_w"):
        assert np.array_equal(bits(bt[k].cpu()), bits(b[k].cpu())), k
    dout = synthetic.normal_bf16(T, s.H, 1.0, 7, "fill").to(DEV)
    args = (cfg, d["x"], d["w_router"], d["w13"], d["w2"], bt["logits"], bt["topk_ids"],
            bt["topk_w"], dout)
    g0 = moe.backward(*args, token_mask=mask, w13_s=d["w13_s"], w2_s=d["w2_s"], keep=True)
    g1 = moe.backward(*args, token_mask=mask, w13_s=d["w13_s"], w2_s=d["w2_s"], keep=True,
                      ws=ws, saved=True)
    torch.cuda.synchronize()
    for k, v in g0.items():
        if v is not None:
            assert np.array_equal(bits(g1[k].cpu()), bits(v.cpu())), k

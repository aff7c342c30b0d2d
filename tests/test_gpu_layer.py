"""Whole-layer parity at the pages' layer shapes, through the C ABI:

* level 1 (bit-exact): routes and weights against the oracle given the GPU's fp32
  logits, the dispatch indices, and the combine given the GPU's expert outputs;
* level 2 (tolerance): router logits, expert outputs and the bf16 layer output against
  the FP64 oracle on sampled tokens (row max relative error <= 1e-2, mean abs reported);
* the one-call moe_forward equals the stage-by-stage composition bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from deterministic_invariant_routing_b200 import moe, synthetic
from helpers import (DEV, LEVEL2_ROW_REL, REPORT, bits, expert_subset, layer, mean_abs_err,
                     near_tie_count, reference_rows, row_rel_err)

pytestmark = pytest.mark.gpu


def run_stages(cfg, d, mask=None):
    logits, ids, w = moe.route(cfg, x=d["x"], w_router=d["w_router"], logit_bias=d["logit_bias"],
                               sel_bias=d["sel_bias"], token_mask=mask, check=False)
    offsets, perm_token, dest_row, x_perm = moe.permute(cfg, ids, x=d["x"])
    y, ys = moe.grouped_ffn(cfg, d["x"], x_perm, perm_token, offsets, d["w13"], d["w2"],
                            d["w13_s"], d["w2_s"])
    out = moe.combine(cfg, y, w, dest_row, ys, mask)
    torch.cuda.synchronize()
    return dict(logits=logits, ids=ids, w=w, offsets=offsets, perm_token=perm_token,
                dest_row=dest_row, x_perm=x_perm, y=y, ys=ys, out=out)


def sample_tokens(T, n, seed):
    rng = np.random.default_rng(seed)
    edge = [0, 1, 2, T - 3, T - 2, T - 1]
    pick = rng.choice(T, size=min(n, T), replace=False)
    return np.unique(np.clip(np.concatenate([edge, pick]), 0, T - 1)).astype(np.int32)


def check_layer(name, T, n_sample=16, keep=None, report=None, **over):
    s, d, cfg = layer(name, T, **over)
    mask = None
    if keep is not None:
        mask = synthetic.random_mask(T, keep, 77).to(DEV)
    r = run_stages(cfg, d, mask)
    mask_np = None if mask is None else mask.cpu().numpy()
    x_cpu = d["x"].cpu()
    sel = sample_tokens(T, n_sample, T)

    # router logits: fp32 tensor-core accumulation vs FP64
    wr_cpu = d["w_router"].cpu()
    lb = None if d["logit_bias"] is None else d["logit_bias"].cpu()
    l64 = oracle.logits64(x_cpu[sel], wr_cpu, lb)
    xf = x_cpu[sel].float().numpy().astype(np.float64)
    scale = np.abs(xf) @ np.abs(wr_cpu.float().numpy().astype(np.float64)).T
    g_logits = r["logits"].cpu().numpy()
    assert np.all(np.abs(g_logits[sel] - l64) <= 2e-5 * scale + 1e-6)

    # level 1: routes from the GPU's logits, bit-exact
    sb = None if d["sel_bias"] is None else d["sel_bias"].cpu().numpy()
    r_ids, r_w, r_st = oracle.route_fp32(g_logits, s.K, s.score_fn, s.renorm, s.route_scale,
                                         sel_bias=sb, mask=mask_np, n_group=s.n_group,
                                         topk_group=s.topk_group)
    g_ids = r["ids"].cpu().numpy()
    assert np.array_equal(g_ids, r_ids)
    assert np.array_equal(r["w"].cpu().numpy().view(np.uint32), r_w.view(np.uint32))
    assert r_st.tolist() == [0, 0]
    # dispatch, bit-exact
    r_off, r_perm, r_dest, _ = oracle.permute(r_ids, s.E)
    assert np.array_equal(r["offsets"].cpu().numpy(), r_off)
    n_rows = int(r_off[-1])
    assert np.array_equal(r["perm_token"].cpu().numpy()[:n_rows], r_perm[:n_rows])
    assert np.array_equal(r["dest_row"].cpu().numpy(), r_dest)
    # combine given the GPU's expert outputs, bit-exact (every token)
    ys = r["ys"]
    ref_out_bits = oracle.combine_fp32(bits(r["y"]), r["w"].cpu(), r_dest,
                                       None if ys is None else bits(ys), mask_np)
    assert np.array_equal(bits(r["out"]), ref_out_bits)

    # level 2: expert outputs of sampled rows vs FP64
    rng = np.random.default_rng(5)
    rows = rng.choice(n_rows, size=min(12, n_rows), replace=False) if n_rows else []
    for row in rows:
        t = int(r_perm[row])
        e = int(np.searchsorted(r_off, row, side="right") - 1)
        y64 = oracle.expert_ffn64(x_cpu[t], d["w13"][e].cpu(), d["w2"][e].cpu())
        err = np.abs(r["y"][row].float().cpu().numpy() - y64).max() / np.abs(y64).max()
        assert err <= LEVEL2_ROW_REL, (row, t, e, err)
    if ys is not None:
        for t in sel[:6]:
            y64 = oracle.expert_ffn64(x_cpu[t], d["w13_s"].cpu(), d["w2_s"].cpu())
            err = np.abs(ys[t].float().cpu().numpy() - y64).max() / np.abs(y64).max()
            assert err <= LEVEL2_ROW_REL
    # level 2: layer output of sampled tokens vs the FP64 layer on the same routes
    l64_sel = l64
    ref = reference_rows(s, d, x_cpu[sel], l64_sel, r_ids[sel],
                         None if mask_np is None else mask_np[sel])
    g_out = r["out"][torch.from_numpy(sel).long().to(DEV)]
    live = np.abs(ref).max(axis=1) > 0
    errs = row_rel_err(g_out, ref)
    assert np.all(errs[live] <= LEVEL2_ROW_REL), errs
    if mask_np is not None:
        assert np.all(bits(r["out"])[mask_np == 0] == 0)

    # the gather fused into the GEMM's operand loads gives the same expert outputs
    y_g, ys_g = moe.grouped_ffn(cfg, d["x"], None, r["perm_token"], r["offsets"], d["w13"],
                                d["w2"], d["w13_s"], d["w2_s"])
    assert np.array_equal(bits(y_g[:n_rows]), bits(r["y"][:n_rows]))

    # the one-call forward is the same computation
    out1, b = moe.forward(cfg, d["x"], d["w_router"], d["w13"], d["w2"],
                          logit_bias=d["logit_bias"], sel_bias=d["sel_bias"], token_mask=mask,
                          w13_s=d["w13_s"], w2_s=d["w2_s"], keep=True)
    assert np.array_equal(bits(out1), bits(r["out"]))
    assert np.array_equal(bits(b["logits"]), bits(r["logits"]))
    assert np.array_equal(b["topk_ids"].cpu().numpy(), g_ids)
    rep = dict(max_row_rel=float(errs[live].max()) if live.any() else 0.0,
               mean_abs=mean_abs_err(g_out, ref), tokens=int(sel.size),
               near_ties=near_tie_count(g_logits[sel], s, sb))
    REPORT.append(f"level 2 {name} T={T}{'' if keep is None else f' keep={keep}'}"
                  f"{''.join(f' {k}={v}' for k, v in over.items())}: "
                  f"max row rel err {rep['max_row_rel']:.3e}, mean abs err "
                  f"{rep['mean_abs']:.3e} over {rep['tokens']} sampled tokens, "
                  f"{rep['near_ties']} near ties among them")
    if report is not None:
        report.update(rep)
    return r


def test_tiny():
    check_layer("tiny", 64, n_sample=64)


def test_tiny_masked():
    check_layer("tiny", 64, n_sample=64, keep=0.7)


def test_tiny_single_token():
    check_layer("tiny", 1)


def test_tiny_ragged():
    check_layer("tiny", 333, n_sample=40)


@pytest.mark.parametrize("T", [1, 64, 4096, 16384])
def test_qwen3_30b_a3b_shape(T):
    check_layer("qwen3_30b_a3b", T, n_sample=16)


def expert_edge_rows(off):
    """Per expert: its first and last row, every row of its last partial 32-row block
    (stored from registers, not through a TMA store tile) and every row of a short tail of
    1..128 rows past its last full 256-row tile (computed by the one-SM tail kernel)."""
    rows = set()
    for e in range(off.size - 1):
        a, n = int(off[e]), int(off[e + 1] - off[e])
        if n == 0:
            continue
        rows |= {a, a + n - 1}
        rows |= set(range(a + n - n % 32, a + n))
        if 0 < n % 256 <= 128:
            rows |= set(range(a + n - n % 256, a + n))
    return np.array(sorted(rows), np.int64)


def test_qwen3_30b_a3b_expert_edge_rows_T16384():
    """Level 2 at the bench size on the rows where a kernel's bookkeeping could go wrong
    without a sampled row noticing: every expert's first and last row, its partial 32-row
    block and its short tail (see expert_edge_rows), each expert output row against the
    FP64 expert FFN of its token (row max relative error <= 1e-2)."""
    from oracle import backward64 as B
    T = 16384
    s, d, cfg = layer("qwen3_30b_a3b", T)
    r = run_stages(cfg, d)
    off = r["offsets"].cpu().numpy()
    perm = r["perm_token"].cpu().numpy()
    rows = expert_edge_rows(off)
    x64 = B.bf16_to_f64(bits(d["x"]))
    y_g = r["y"].float().cpu().numpy().astype(np.float64)
    worst, n_tail, errs = 0.0, 0, []
    for e in range(s.E):
        rr = rows[(rows >= off[e]) & (rows < off[e + 1])]
        if rr.size == 0:
            continue
        n = int(off[e + 1] - off[e])
        n_tail += (n % 256) if 0 < n % 256 <= 128 else 0
        _, _, _, y64 = B._experts_forward(x64[perm[rr]], B.bf16_to_f64(bits(d["w13"][e])),
                                          B.bf16_to_f64(bits(d["w2"][e])))
        rel = np.abs(y_g[rr] - y64).max(axis=1) / np.abs(y64).max(axis=1)
        assert np.all(rel <= LEVEL2_ROW_REL), (e, rr[np.argmax(rel)], rel.max())
        errs.append(np.abs(y_g[rr] - y64).mean())
        worst = max(worst, float(rel.max()))
    REPORT.append(f"level 2 qwen3_30b_a3b T={T} expert edge rows: {rows.size} rows "
                  f"({n_tail} in short tails) max row rel err {worst:.3e}, mean abs err "
                  f"{float(np.mean(errs)):.3e}")


def test_qwen3_30b_a3b_masked():
    check_layer("qwen3_30b_a3b", 4096, n_sample=16, keep=0.8)


def test_dspark_shape():
    check_layer("dspark", 8192, n_sample=16)


def test_dsv_sigmoid_shape():
    check_layer("dsv_sigmoid", 8192, n_sample=12)


def test_dsv_sqrtsoftplus_shape():
    """The DeepSeek-style layer with sqrtsoftplus scores (level 1 bit-exact routes from the
    GPU's logits, level 2 outputs against FP64 sqrt(softplus) weights)."""
    check_layer("dsv_sigmoid", 4096, n_sample=12, score_fn=synthetic.SQRTSOFTPLUS)


def test_dsv_sigmoid_group_limited():
    """The DeepSeek-style layer with group-limited selection (8 groups of 32, 4 kept)."""
    r = check_layer("dsv_sigmoid", 4096, n_sample=12, n_group=8, topk_group=4)
    ids = r["ids"].cpu().numpy()
    assert np.all(np.array([len(set(row // 32)) for row in ids]) <= 4)


def test_tied_router_rows_pick_lower_id():
    """Two experts with identical router rows tie exactly on every token; the lower id
    must come first (tiny layer, x-mode, 4 duplicated token pairs)."""
    s, d, cfg = layer("tiny", 64)
    d["w_router"][5] = d["w_router"][2]
    for a, b in ((0, 1), (10, 11), (20, 30), (40, 63)):
        d["x"][b] = d["x"][a]
    r = run_stages(cfg, d)
    lg = r["logits"].cpu().numpy()
    assert np.array_equal(lg[:, 5].view(np.uint32), lg[:, 2].view(np.uint32))
    ids = r["ids"].cpu().numpy()
    assert np.all((ids == 2).any(1) | ~(ids == 5).any(1))  # 5 never without 2
    both = (ids == 2).any(1) & (ids == 5).any(1)
    for t in np.flatnonzero(both):
        row = list(ids[t])
        assert row.index(2) < row.index(5)
    ob = bits(r["out"])
    for a, b in ((0, 1), (10, 11), (20, 30), (40, 63)):
        assert np.array_equal(ids[a], ids[b]) and np.array_equal(ob[a], ob[b])


@pytest.mark.parametrize("E,H,T", [(33, 128, 300), (100, 2048, 1000), (300, 1024, 257),
                                   (1024, 8192, 130), (8, 4096, 513), (256, 4096, 129)])
def test_router_logits_odd_shapes(E, H, T):
    """The router product at expert counts and hidden sizes the layer shapes do not reach:
    column tiles of 64, 128 and 256 experts with part of the last one past E, one or several
    column tiles, K split over clusters of 1, 2 and 8 CTAs (and the CTA-pair path at
    E = 256), ragged last row tiles. Every token's logits against the FP64 product within
    the same bound as the layer tests; the logit bias added after the K reduction."""
    rng = np.random.default_rng(E * 7 + H)
    x = synthetic.normal_bf16(T, H, 1.0, E + H, "x")
    wr = synthetic.normal_bf16(E, H, 0.02, E + H, "w_router")
    lb = torch.from_numpy(rng.normal(0, 0.5, E).astype(np.float32))
    cfg = moe.Config(T=T, H=H, E=E, K=1, I=128)
    logits, _, _ = moe.route(cfg, x=x.to(DEV), w_router=wr.to(DEV), logit_bias=lb.to(DEV),
                             check=False)
    torch.cuda.synchronize()
    g = logits.cpu().numpy()
    ref = oracle.logits64(x, wr, lb)
    xf = x.float().numpy().astype(np.float64)
    scale = np.abs(xf) @ np.abs(wr.float().numpy().astype(np.float64)).T
    assert g.shape == (T, E)
    assert np.all(np.abs(g - ref) <= 2e-5 * scale + 1e-6)
    # the same tokens in another batch give the same bits (the split depends on H only)
    sub = x[T // 3:T // 3 + 5].clone()
    cfg5 = moe.Config(T=5, H=H, E=E, K=1, I=128)
    l5, _, _ = moe.route(cfg5, x=sub.to(DEV), w_router=wr.to(DEV), logit_bias=lb.to(DEV),
                         check=False)
    torch.cuda.synchronize()
    assert np.array_equal(bits(l5), bits(logits[T // 3:T // 3 + 5]))

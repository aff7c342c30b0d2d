"""The oracle against the hand-worked two-token example (tests/golden)."""
import numpy as np

import oracle


def test_two_token_example(golden):
    g = golden("two_token_route_combine.json")
    logits = np.array(g["logits"], np.float32)
    bias = np.array(g["sel_bias"], np.float32)
    ids, w, st = oracle.route_fp32(logits, g["K"], oracle.SOFTMAX, g["renorm"],
                                   g["route_scale"], sel_bias=bias)
    assert ids.tolist() == g["expect_ids"]
    assert w.tolist() == g["expect_w"]
    assert st.tolist() == [0, 0]
    offsets, perm_token, dest_row, bad = oracle.permute(ids, g["E"])
    assert offsets.tolist() == g["expect_offsets"]
    assert dest_row.tolist() == g["expect_dest_row"]
    assert perm_token[:offsets[-1]].tolist() == g["expect_perm_token"]
    y = oracle.f32_to_bf16(np.array(g["y"], np.float32))
    ys = oracle.f32_to_bf16(np.array(g["y_shared"], np.float32))
    assert np.array_equal(oracle.bf16_to_f32(y), np.array(g["y"], np.float32))
    out = oracle.combine_fp32(y, w, dest_row, ys)
    assert [[f"{v:04x}" for v in row] for row in out] == g["expect_out_bf16_hex"]

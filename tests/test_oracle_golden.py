"""The oracle reproduces its frozen regression fixture (tests/golden)."""
import json
import os

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_frozen_fixture():
    with open(os.path.join(HERE, "golden", "oracle_tiny.json")) as f:
        g = json.load(f)
    inp = {k: np.array(v) for k, v in g["inputs"].items()}
    for causal, key in ((False, "attn_dense"), (True, "attn_causal")):
        want = g["cases"][key]
        o, l = oracle.attention_forward(inp["q"], inp["k"], inp["v"], causal)
        dq, dk, dv = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["dout"], causal)
        for name, got in (("out", o), ("lse", l), ("dq", dq), ("dk", dk), ("dv", dv)):
            np.testing.assert_allclose(got, np.array(want[name]), atol=1e-13, err_msg=name)
    want = g["cases"]["s2_g4_shift2_causal"]
    o, l = oracle.s2attn_forward(inp["s2_q"], inp["s2_k"], inp["s2_v"], 4, 2, True)
    np.testing.assert_allclose(o, np.array(want["out"]), atol=1e-13)
    np.testing.assert_allclose(l, np.array(want["lse"]), atol=1e-13)
    want = g["cases"]["packed_causal"]
    o, l = oracle.packed_attention_forward(inp["q"][0], inp["k"][0], inp["v"][0], want["cu"], True)
    np.testing.assert_allclose(np.nan_to_num(o, nan=0.0), np.array(want["out"]), atol=1e-13)
    np.testing.assert_allclose(np.nan_to_num(l, nan=0.0), np.array(want["lse"]), atol=1e-13)
    want = g["cases"]["ffn_block2"]
    args = (inp["ffn_x"], inp["ffn_w_gate"], inp["ffn_w_up"], inp["ffn_w_down"])
    np.testing.assert_allclose(oracle.ffn_forward(*args, block=2), np.array(want["out"]),
                               atol=1e-13)
    got = oracle.ffn_backward(*args, inp["ffn_dout"], block=2)
    for name, a in zip(("dx", "dw_gate", "dw_up", "dw_down"), got):
        np.testing.assert_allclose(a, np.array(want[name]), atol=1e-12, err_msg=name)

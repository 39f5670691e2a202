"""Writes tests/golden/oracle_tiny.json: a frozen oracle result on a tiny
fixed input, so an unintended change to the oracle's arithmetic shows up.

The pages print no worked attention example, so no fixture here carries
values from them; this script calls only ``oracle/`` and the seeded numpy
generator below.  Run from the repository root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def build():
    rng = np.random.default_rng(20231002)
    S, Hq, Hkv, d = 8, 4, 2, 4
    q = np.round(rng.standard_normal((1, S, Hq, d)), 3)
    k = np.round(rng.standard_normal((1, S, Hkv, d)), 3)
    v = np.round(rng.standard_normal((1, S, Hkv, d)), 3)
    do = np.round(rng.standard_normal((1, S, Hq, d)), 3)
    cases = {}
    for causal in (False, True):
        o, l = oracle.attention_forward(q, k, v, causal)
        dq, dk, dv = oracle.attention_backward(q, k, v, do, causal)
        cases["attn_causal" if causal else "attn_dense"] = dict(
            out=o.tolist(), lse=l.tolist(), dq=dq.tolist(), dk=dk.tolist(), dv=dv.tolist())
    qs = np.round(rng.standard_normal((1, S, Hq, d)), 3)
    ks = np.round(rng.standard_normal((1, S, Hq, d)), 3)
    vs = np.round(rng.standard_normal((1, S, Hq, d)), 3)
    o, l = oracle.s2attn_forward(qs, ks, vs, 4, 2, True)
    cases["s2_g4_shift2_causal"] = dict(out=o.tolist(), lse=l.tolist())
    # drawn after the cases above, so their inputs do not move
    cu = [0, 3, 3, 8]                      # packed: lengths 3, 0, 5 over 8 tokens
    o, l = oracle.packed_attention_forward(q[0], k[0], v[0], cu, True)
    cases["packed_causal"] = dict(cu=cu, out=np.nan_to_num(o, nan=0.0).tolist(),
                                  lse=np.nan_to_num(l, nan=0.0).tolist())
    T, h, f = 5, 4, 6
    fx = np.round(rng.standard_normal((T, h)), 3)
    fg = np.round(rng.standard_normal((f, h)) * 0.5, 3)
    fu = np.round(rng.standard_normal((f, h)) * 0.5, 3)
    fd = np.round(rng.standard_normal((h, f)) * 0.5, 3)
    fdo = np.round(rng.standard_normal((T, h)), 3)
    out = oracle.ffn_forward(fx, fg, fu, fd, block=2)
    dx, dwg, dwu, dwd = oracle.ffn_backward(fx, fg, fu, fd, fdo, block=2)
    cases["ffn_block2"] = dict(out=out.tolist(), dx=dx.tolist(), dw_gate=dwg.tolist(),
                               dw_up=dwu.tolist(), dw_down=dwd.tolist())
    return dict(
        note="oracle regression fixture; values written by this script from oracle/",
        inputs=dict(q=q.tolist(), k=k.tolist(), v=v.tolist(), dout=do.tolist(),
                    s2_q=qs.tolist(), s2_k=ks.tolist(), s2_v=vs.tolist(),
                    ffn_x=fx.tolist(), ffn_w_gate=fg.tolist(), ffn_w_up=fu.tolist(),
                    ffn_w_down=fd.tolist(), ffn_dout=fdo.tolist()),
        cases=cases)


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(path, "w") as f:
        json.dump(build(), f, indent=None, separators=(",", ":"))
    print("wrote", path)

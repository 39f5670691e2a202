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
    return dict(
        note="oracle regression fixture; values written by this script from oracle/",
        inputs=dict(q=q.tolist(), k=k.tolist(), v=v.tolist(), dout=do.tolist(),
                    s2_q=qs.tolist(), s2_k=ks.tolist(), s2_v=vs.tolist()),
        cases=cases)


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(path, "w") as f:
        json.dump(build(), f, indent=None, separators=(",", ":"))
    print("wrote", path)

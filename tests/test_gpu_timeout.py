"""Bounded waits: a forward given a one-clock wait budget must stop, report
LCA_ERR_TIMEOUT through lca_check, and leave the context usable (the next
call with the default budget is correct).  No fault, trap or endless wait:
the kernel unwinds by itself (it lets its in-flight copies and MMAs land,
frees its tensor memory and returns)."""

import pytest
import torch

import oracle
from long_context_exact_attention_b200 import lca
from long_context_exact_attention_b200.inputs import WORKLOADS, make_inputs, shrink

from gpu_util import assert_fwd_close, host

pytestmark = pytest.mark.gpu


def test_wait_budget_runs_out_and_context_survives():
    w = shrink(WORKLOADS["llama2_7b_s32k"], B=1, Hq=2, Hkv=2, S=1024, rope=False, seed=51)
    x = make_inputs(w, "cuda", with_dout=False)
    lca.check()                                   # clear any earlier state
    lca.attn_fwd(x["q"], x["k"], x["v"], causal=True, kv_chunk=256, timeout_cycles=1)
    with pytest.raises(lca.LcaError) as e:
        lca.check()
    assert e.value.status == 4
    lca.check()                                   # the error word was cleared
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=True, kv_chunk=256)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], True)
    assert_fwd_close(host(out), host(lse), ro, rl)

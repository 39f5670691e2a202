"""CPU fp64 oracle for exact long-context attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or run anything here.
The product path (``long_context_exact_attention_b200`` and its CUDA
library) never imports this package, and this package never imports the
product path: the two share no code.

What it computes is the plain definition the pages fix, written out in
numpy float64 with no blocking, fusion or reordering beyond row blocks that
bound memory:

* ``attention``  -- softmax(Q K^T / sqrt(d) + mask) V, its log-sum-exp and its
  analytic gradients ("Attention stays exact": Ring Attention with Blockwise
  Transformers for Near-Infinite Context, Summary; full attention with no
  approximations: sourcepulse project card of the 1M-context training
  recipe, How It Works); and the partial result of one query block over one
  key/value block at given positions, as a host of the ring computes it.
* ``s2attn``     -- LongLoRA's shifted sparse attention taken literally:
  shift half the heads by half a group, split into groups, attend inside
  each group, shift back (LongLoRA: Efficient Fine-tuning of Long-Context
  Large Language Models, Summary).
* ``packed``     -- a packed batch of variable-length sequences: each
  sequence is an independent problem, so the definition applied per slice.
* ``ffn``        -- the blockwise feedforward (gated SiLU, Llama's) computed
  a block of token rows at a time (Ring Attention, Summary and Key points).
* ``merge``      -- the (O, lse) combination of partial results over key
  chunks, whose order does not matter (Ring Attention, Summary).
* ``brute``      -- pure-Python loops on tiny inputs, an independent
  restatement used to pin the vectorised code.

Every function is pinned by ``tests/test_oracle_pins.py`` (closed forms,
invariants, brute force, finite differences, special cases).  No function
here is "parity unpinned".
"""

from .attention import (attention_forward, attention_rows, attention_backward,
                        attention_backward_rows, block_attention, chunked_attention_forward)
from .s2attn import s2attn_forward, s2attn_backward, s2_token_of_position
from .merge import lse_merge
from .packed import packed_attention_forward, packed_attention_backward
from .ffn import ffn_forward, ffn_backward, ffn_backward_columns, ffn_rows, silu

__all__ = [
    "attention_forward", "attention_rows", "attention_backward",
    "attention_backward_rows", "block_attention",
    "chunked_attention_forward", "s2attn_forward", "s2attn_backward",
    "s2_token_of_position", "lse_merge", "packed_attention_forward",
    "packed_attention_backward", "ffn_forward", "ffn_backward", "ffn_backward_columns", "ffn_rows", "silu",
]

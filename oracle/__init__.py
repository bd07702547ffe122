"""fp64 CPU oracle for blockwise attention with online-softmax merging.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
package: only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library (``blockwise_long_context_b200``) and never imports it.

The oracle is written from these pages:

* "Ring Attention with Blockwise Transformers for Near-Infinite Context"
  (pith.science citation hub, abstract): attention computed block by block
  over the key/value sequence, exactly, without approximation.
* "LV-XAttn: Distributed Cross-Attention for Long Visual Inputs in Multimodal
  Large Language Models" (pith.science review page): "The reading" and
  "What carries the argument" (key/value blocks stay put, partial outputs O_i
  and softmax statistics L_i are rescaled and combined as in FlashAttention),
  Figure 3 / Algorithm 1 (O_i, L_i initialised to the empty result and
  updated once per block), "Assumptions" (the online-softmax rescaling is
  exact), the referee report's first major comment (the backward pass is
  not specified; checked here against the exact formula's gradient), and
  Figure 1 / the activation-recomputation passage (K = y W_k, V = y W_v from
  one shared copy of the visual features y, and the gradients of that map).

Every function is pinned by tests under ``tests/`` against closed forms,
invariants, brute force on tiny inputs and an independent library routine
(torch's fp64 scaled-dot-product attention and autograd).  Parity pinned:
all functions; none is "parity unpinned".
"""

from .attention import (  # noqa: F401
    kv_block_bounds,
    attention_fwd,
    attention_probs,
    block_partials,
    merge_partials,
    attention_bwd,
    attention_bwd_keys,
    attention_bwd_rows,
    kv_recompute,
    kv_recompute_bwd,
)

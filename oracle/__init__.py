"""Float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference legs may import anything here.  The
library under ``scaled_dot_product_prefill_b200`` never imports it, and this
package imports nothing from that library: the two share no arithmetic.

The oracle is the plain definition, written out with no tiling, no online
softmax and no reordering beyond what the definition states:

    O = softmax(Q K^T * scale + mask) V

Sources, cited by short key throughout:

[AFS]  "Attention From Scratch -- open-source project and system docs"
       (2048ai.net), sections "Scaled Dot-Product Attention", "Grouped Query
       Attention", "KV Cache", "Flash Attention", "Paged KV Cache" and
       "Quick start / using the source".
[AME]  "Attention mechanism explained: from Self-Attention to Multi-Query
       Attention" (guijiagi.com), sections 2.1 (formula), 2.2 (computation
       flow), 5.2 (GQA implementation), 6 (complexity), 7 (Flash Attention).
[LCT]  "LLM core technology: implementing and optimising Attention"
       (zeeklog.com), sections "GQA implementation logic", "Sliding Window
       Attention", "FlashAttention", "PagedAttention".
[EMHA] Walkthrough of the nine causal-MHA implementations of
       LLMs-from-scratch ch03/02_bonus_efficient-multihead-attention
       (gsyq.cn), sections 3.1-3.9, 4.1, 4.2, 5.
[ANAT] "Taking LLMs apart (2): attention by hand" (blog.kerro.cn), sections
       "softmax", "sqrt(d) is not decoration" (scale table), "full
       implementation" / causal mask / pitfalls 1-4, "KV cache" (timing,
       FLOP and byte tables), "GQA / MLA", "FlashAttention".

Modules:

* ``sdpa``  -- numpy float64: visibility predicate, weights, attention,
  sampled rows, paged gather and paged decode.
* ``brute`` -- pure-Python loops with ``math.exp``: an independent second
  statement of the same definition for tiny shapes.
* ``fp8``   -- the value of each FP8 E4M3 code, for the 8-bit paged cache
  (decoded, then fed to ``sdpa`` like any other cache).

Every function is pinned by ``tests/test_oracle_pins.py`` against closed
forms, invariants and the values the pages print (``tests/golden/``); none
is "parity unpinned".
"""
from . import brute, fp8, sdpa  # noqa: F401

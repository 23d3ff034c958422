"""Plain fp64 CPU oracle for exact blockwise ring attention and the blockwise FFN.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this package:
only the test-suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library (no kernels, headers, helpers, tables or constants) and imports
nothing from ``exact_blockwise_long_b200``.

What it computes follows the pages on Ring Attention:

* "Ring Attention with Blockwise Transformers for Near-Infinite Context"
  (paper abstract): blockwise self-attention and feed-forward, exact, "without
  resorting to approximations".
* chapterpal keyword page "Ring Attention" (definition paragraph): the
  sequence is partitioned into blocks, each block keeps its queries while the
  key/value blocks circulate around a ring.
* darcstar.tech research note on the same paper, "DarcStar commentary",
  paragraphs one and two: online softmax is associative, partial attention of
  separate shards combines exactly; the causal mask and the softmax
  denominator must be combined across chunks exactly.

Every function here is either the plain mathematical definition (full-matrix
softmax attention, its gradient, a SwiGLU feed-forward) or the method's steps
written out in the pages' terms (shards, ring order, chunk tiles, log-sum-exp
merge) for pinning the definition against the method.

Parity status per function (what pins it is in ``tests/test_oracle.py``):

* ``attention_forward``          pinned (hand-derived golden values, closed
                                 forms, brute force, scipy softmax/logsumexp)
* ``attention_backward``         pinned (central finite differences, shift and
                                 homogeneity invariants)
* ``attention_forward_gqa`` / ``attention_backward_gqa``
                                 pinned (one key/value head per query head
                                 reduces to the pinned plain functions; MQA
                                 closed form; finite differences)
* ``attention_decode``           pinned (the last row of causal attention
                                 over the same keys; q = 0 closed form)
* ``ring_blockwise_forward``     pinned (equals the full matrix for every S
                                 and chunk size, order invariant)
* ``lse_merge``                  pinned (closed form of two-part softmax,
                                 associativity, neutral element)
* ``attention_rows`` / ``attention_head_rows`` /
  ``attention_backward_key_rows`` /
  ``attention_backward_query_rows``
                                 pinned (equal to the full functions on the
                                 sampled subset)
* ``swiglu_ffn`` / ``blockwise_ffn``
                                 pinned (zero inputs, chunk invariance,
                                 explicit loop, scipy expit)
* ``swiglu_ffn_backward`` / ``blockwise_ffn_backward``
                                 pinned (central finite differences of
                                 sum(dy * y), zero-weight closed forms, chunk
                                 invariance, linearity in dy)
* ``swiglu_ffn_backward_terms``  error-bound helper (sums of |term|), pinned
                                 by dominating |gradient| element-wise
* ``rmsnorm`` / ``rmsnorm_backward``
                                 pinned (unit mean square with g = 1, scale
                                 invariance, constant rows, finite differences)
* ``layer_forward`` / ``layer_backward``
                                 pinned (central finite differences of every
                                 parameter and input; wo = w2 = 0 closed form;
                                 causal locality and batch independence)
"""

from .attention import (  # noqa: F401
    attention_forward,
    attention_backward,
    attention_forward_gqa,
    attention_backward_gqa,
    attention_decode,
    ring_blockwise_forward,
    ring_blockwise_step,
    lse_merge,
    attention_rows,
    attention_head_rows,
    attention_backward_query_rows,
    attention_backward_key_rows,
    ring_visit_order,
    ring_visit_order_bwd,
)
from .ffn import (  # noqa: F401
    swiglu_ffn,
    blockwise_ffn,
    silu,
    sigmoid,
    swiglu_ffn_backward,
    blockwise_ffn_backward,
    swiglu_ffn_backward_terms,
)
from .layer import (  # noqa: F401
    PARAM_NAMES,
    layer_backward,
    layer_forward,
    rmsnorm,
    rmsnorm_backward,
)

"""CPU oracle for the MTGR HSTU-block forward — TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 NumPy restatement of what the MTGR pages define: the
user-aggregated sample D = [U, S, R, [C,I]_1..K], Group-Layer Normalization, the
three-rule dynamic mask, pointwise SiLU attention normalised by the user's token
count, the U gate, the second GroupLN and the MLP with residual (MTGR paper,
"Method", the block update equations; fun-rec chapter 7.3, sections 7.3.3
"Group Layer Normalization" and 7.3.4 "Dynamic Masking"); and, on either side
of the stack, the per-domain token MLPs and the CTR/CTCVR heads (``tokens.py``).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package. The CUDA library never links, imports or
calls it, and it shares no code with the CUDA library.

Parity pins: every function here is checked in ``tests/test_oracle_*.py``
against hand-derived expected values (``tests/golden/``), library routines on
special cases, closed forms and invariants. Absolute numeric values of the full
model are pinned only by these definitions: the pages print no worked numeric
example, weights or activations (parity unpinned against the pages' numbers).
"""

from .mtgr import (  # noqa: F401
    EPS,
    BM,
    BN,
    silu,
    pack_offsets,
    user_mask,
    group_layernorm,
    group_layernorm_pooled,
    VARIANT_POOLED_GLN,
    VARIANT_SILU_QKVU,
    VARIANT_RAB,
    RAB_MAX_DIST,
    RAB_TIME_BUCKETS,
    rab_time_bucket,
    rab_bias,
    hstu_attention,
    hstu_block,
    hstu_stack,
    mask_meta,
    visible_pairs,
)
from .backward import hstu_block_backward  # noqa: F401
from .tokens import (  # noqa: F401
    token_mlp,
    tokenize,
    candidate_heads,
)

"""fp64 CPU oracle for exact softmax attention (prefill, paged decode, MLA decode, backward).

TEST INFRASTRUCTURE ONLY. This package is the slow, plain definition that the
CUDA path is checked against. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and its ``--impl reference`` arm) may
import it. The product path (``exact_softmax_attention_causal_b200``) never
imports, calls or links anything here, and nothing here imports the product
path: the two share no code.

Every function cites the passage of the source pages it follows. All of them
are pinned by ``tests/test_oracle_pins*.py`` against values and identities the
pages and the mathematics fix; none is "parity unpinned".
"""

from .attention import (  # noqa: F401
    MASK_FULL,
    MASK_CAUSAL,
    MASK_SLIDING_WINDOW,
    allowed_mask,
    sdpa_rows,
    prefill_ref,
    prefill_rows_ref,
    prefill_paged_ref,
    gather_paged_ref,
    decode_paged_ref,
    decode_rows_ref,
    lse_merge_ref,
    kv_cache_bytes,
)
from .mla import mla_cache_bytes, mla_decode_ref, mla_decode_rows_ref  # noqa: F401
from .backward import prefill_backward_ref, sdpa_backward_rows  # noqa: F401

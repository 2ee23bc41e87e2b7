"""CPU float64 oracle for the fused scaled-dot-product attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
link anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code, header, table or helper with the CUDA library under
``tiled_attention_13_b200/``; the only module both sides see is the seeded
input generator ``tiled_attention_13_b200/inputs.py``, which holds no
attention arithmetic.

Every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle.py`` (closed forms, invariants, 50-digit brute force, the
pages' printed facts); none is "parity unpinned".
"""

from .attention_ref import (  # noqa: F401
    attention,
    attention_batched,
    attention_rows,
    attention_tiled_online,
    online_softmax_step,
    resolve_scale,
    allowed_keys,
    attention_paged,
    gather_paged_kv,
    merge_partials,
    band_mask,
    block_sparse_mask,
    attention_masked,
)
from .backward_ref import (  # noqa: F401
    attention_backward,
    attention_backward_batched,
    attention_backward_tiled,
)

"""fp64 CPU oracle for PipeFusion patch attention and the guidance combine.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import it.  The CUDA library never
calls it, and it shares no code with the CUDA library: it is a plain, slow, obviously
correct restatement of what the pages define, in float64 numpy.

Modules
-------
attention   plain-definition patch attention (which rows are fresh, which are stale),
            a stateful KV-buffer walk, and the full-attention primitive.
cfg         guidance combine eps_u + w (eps_c - eps_u) and rel-MAE_t.

Parity status: every function here is pinned by ``tests/test_oracle_*.py`` against
closed forms, brute force, reductions to ordinary attention and hand-derived golden
fixtures.  No function is "parity unpinned".
"""
from .attention import (  # noqa: F401
    attend,
    softmax_probs,
    image_key_rows,
    patch_keys,
    patch_attention,
    distrifusion_attention,
    expected_buffer,
    KVBufferWalk,
)
from .cfg import cfg_combine, rel_mae, cfg_combine_relmae  # noqa: F401

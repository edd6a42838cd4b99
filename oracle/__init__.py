"""fp64 CPU oracle (test infrastructure only; see ``gdn_oracle``).

Parity status of each function: every function here is pinned by ``-m "not gpu"`` tests. The
GDN functions are pinned in ``tests/test_oracle_pins.py``, the softmax attention of the hybrid
blocks in ``tests/test_softmax_oracle.py`` and the 3D RoPE in ``tests/test_rope_oracle.py``. The pins are closed forms, invariants,
special cases that reduce to textbook routines, brute force on tiny inputs, and hand-worked
examples under ``tests/golden/``.
"""
from .gdn_oracle import (  # noqa: F401
    e4m3_decode,
    frame_output,
    frame_statistics,
    frame_update,
    frame_update_backward,
    gdn_frame_backward,
    gdn_frame_forward,
    gdn_frame_forward_fp8,
    gdn_frame_step,
    la_block_causal,
)
from .rope_oracle import rope_3d, rope_3d_split  # noqa: F401
from .softmax_oracle import softmax_attention_chunk_causal  # noqa: F401

"""fp64 CPU oracle (test infrastructure only; see ``gdn_oracle``).

Parity status of each function: every function here is pinned by ``-m "not gpu"`` tests. The
GDN functions are pinned in ``tests/test_oracle_pins.py`` and the softmax attention of the
hybrid blocks in ``tests/test_softmax_oracle.py``. The pins are closed forms, invariants,
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
from .softmax_oracle import softmax_attention_chunk_causal  # noqa: F401

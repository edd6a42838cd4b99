"""The fp64 oracle against its pins (CPU only)."""
import types

import pytest

import oracle
from tests import oracle_pins

IMPL = types.SimpleNamespace(
    gdn_frame_forward=oracle.gdn_frame_forward,
    gdn_frame_step=oracle.gdn_frame_step,
    la_block_causal=oracle.la_block_causal,
    frame_statistics=oracle.frame_statistics,
    e4m3_decode=oracle.e4m3_decode,
    gdn_frame_forward_fp8=oracle.gdn_frame_forward_fp8,
    gdn_frame_backward=oracle.gdn_frame_backward,
)


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(IMPL)

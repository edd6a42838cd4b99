"""The benchmark's byte accounting (host logic, CPU only): the algorithmic bytes it divides by
the measured time, counted here independently from the tensor shapes of the 720p clip."""
import gdn_inputs

import bench

W = gdn_inputs.WORKLOADS["720p"]
FH = W.B * W.H * W.T            # frame-heads
TOK = W.N * W.D * 2             # one frame-head of a bf16 token tensor
DD = W.D * W.D
STATE = W.B * W.H * DD * 4


def test_forward_path_bytes():
    # q, k, v read and out written; gamma, beta read; the final state written
    assert bench.algorithmic_bytes(W) == FH * 4 * TOK + W.B * W.T * W.H * 8 + STATE
    assert bench.algorithmic_bytes(W) == 17_320_990_880


def test_backward_path_bytes():
    # q, k, v, dO read and dq, dk, dv written; gamma, beta read and dgamma, dbeta written;
    # S_0 read and dS_0 written
    assert bench.backward_bytes(W) == FH * 7 * TOK + W.B * W.T * W.H * 16 + 2 * STATE
    assert bench.backward_bytes(W) == 30_312_100_160


def test_backward_kernel_bytes():
    assert bench.kernel_bytes("gdn_bwd_token_kernel_dq", W) == FH * (2 * TOK + DD * 2)
    assert bench.kernel_bytes("gdn_bwd_token_kernel_dkdv", W) == FH * (4 * TOK + 2 * DD * 2)
    assert bench.kernel_bytes("gdn_bwd_frame_kernel", W) == FH * (3 * DD * 2 + DD * 4 + DD * 2 + 16)
    assert bench.kernel_bytes("gdn_bwd_chain_kernel", W) == FH * (DD * 8 + 8) + STATE


def test_per_launch_bytes_for_passes_and_segments():
    stats = bench.kernel_bytes("gdn_stats_kernel", W)
    # forward: one launch per step
    assert bench.per_launch_bytes("gdn_stats_kernel", W, False, False, 10, 10) == stats
    # backward: two full statistics passes per step, so each launch moves a full pass
    assert bench.per_launch_bytes("gdn_stats_kernel", W, False, True, 10, 20) == stats
    # a kernel run in 4 segments per step: each launch moves a quarter of the pass
    dkdv = bench.kernel_bytes("gdn_bwd_token_kernel_dkdv", W)
    assert bench.per_launch_bytes("gdn_bwd_token_kernel_dkdv", W, False, True, 20, 80) == dkdv / 4
    assert bench.per_launch_bytes("no_such_kernel", W, False, True, 1, 1) is None

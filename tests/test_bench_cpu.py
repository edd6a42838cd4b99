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


def test_traffic_file_entries():
    """profiles/traffic.json: every entry names a kernel bench.py knows, a capture summary that
    exists, and DRAM bytes per launch that are positive; the 720p fused-kernel entries (captures
    of 96 frames scaled to 961) stay within a few percent of the algorithmic bytes they stand
    for (more would mean re-reads, less a scaling mistake)."""
    import json
    import os
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        kernels = json.load(f)["kernels"]
    for name, entries in kernels.items():
        assert name in bench.KERNEL_SOURCES, name
        for e in entries if isinstance(entries, list) else [entries]:
            assert set(e) >= {"workload", "source_digest", "dram_bytes_per_launch", "capture"}, e
            assert e["dram_bytes_per_launch"] > 0
            capture = e["capture"].split(" ")[0]
            assert os.path.exists(os.path.join(bench.ROOT, capture)), capture
    fused = {e["workload"]: e["dram_bytes_per_launch"] for e in kernels["gdn_fused_kernel"]}
    for workload, fp8 in (("720p", False), ("720p+fp8", True), ("720p+rope", False)):
        ratio = fused[workload] / bench.algorithmic_bytes(W, fp8)
        assert 0.95 <= ratio <= 1.05, (workload, ratio)


def test_traffic_lookup_follows_source_digest(tmp_path, monkeypatch):
    """bench.ncu_traffic reports an entry only for the workload it was taken on and only while the
    kernel's sources hash to the entry's digest."""
    import json
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"kernels": {
        "gdn_step_kernel": {"workload": "stream", "source_digest": "abc",
                            "dram_bytes_per_launch": 123, "capture": "x"},
        "gdn_fused_kernel": [{"workload": "720p", "source_digest": "abc",
                              "dram_bytes_per_launch": 7, "capture": "x"},
                             {"workload": "480p", "source_digest": "old",
                              "dram_bytes_per_launch": 8, "capture": "x"}]}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_digest", lambda kernel=None: "abc")
    assert bench.ncu_traffic("gdn_step_kernel", "stream") == 123
    assert bench.ncu_traffic("gdn_step_kernel", "720p") is None        # other workload
    assert bench.ncu_traffic("gdn_fused_kernel", "720p") == 7
    assert bench.ncu_traffic("gdn_fused_kernel", "480p") is None       # sources changed since
    assert bench.ncu_traffic("gdn_rope_kernel", "720p") is None        # no entry

"""Host-side checks of bench.py's bookkeeping (CPU, no GPU): every workload
has an accounting of its work and bytes, every kernel source is covered by
the hash that guards stored ncu traffic, and every stored traffic figure
points at an existing profile summary."""
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantized_gemm_token_b200", "csrc")


@pytest.mark.parametrize("name", sorted(k for k, w in bench.WORKLOADS.items() if w["kind"] not in ("mma_peak",)))
def test_every_workload_is_accounted(name):
    wl = bench.WORKLOADS[name]
    d = {}
    if wl["kind"] in ("bsr", "bsr_dense"):
        # the BSR accounting reads the block pattern's size only
        import synth
        bs = wl.get("bs", 64)
        M, K, N = 65792, (1280 if wl["layer"] == "fc1" else 5120), (5120 if wl["layer"] == "fc1" else 1280)
        crow, _ = synth.bsr_pattern(N // bs, K // bs, wl.get("keep", 0.10), 3)
        d = dict(M=M, K=K, N=N, crow=crow)
    ops, dom = bench.step_accounting(wl, d)
    assert dom["kernel"] in bench.KERNEL_SOURCES
    assert dom["bytes"] > 0
    if wl["kind"] != "quant":
        assert ops > 0 and dom["ops"] == ops


def test_kernel_sources_cover_every_cuda_file():
    listed = set()
    for files in bench.KERNEL_SOURCES.values():
        for f in files:
            assert os.path.exists(os.path.join(CSRC, f)), f
            listed.add(f)
    on_disk = {f for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))}
    assert on_disk <= listed, on_disk - listed


def test_stored_traffic_points_at_profiles():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    for wl, entries in t.items():
        if wl.startswith("_"):
            continue
        assert wl in bench.WORKLOADS
        for kernel, e in entries.items():
            assert kernel in bench.KERNEL_SOURCES
            assert e["bytes_per_launch"] == e["read"] + e["write"]
            assert os.path.exists(os.path.join(ROOT, "profiles", e["from"]))
            # a figure taken on other sources is reported as null by the bench
            if e["source_hash"] != bench.kernel_source_hash(kernel):
                assert bench.measured_traffic(wl, kernel) is None
            else:
                assert bench.measured_traffic(wl, kernel) == e["bytes_per_launch"]

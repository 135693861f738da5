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


def test_write_floor_is_the_slower_of_write_and_copy():
    """_hbm_entry's floor: the output at the measured write-only rate, or all
    bytes at the copy rate, whichever takes longer; frac_vs_floor = floor /
    measured time."""
    peaks = dict(hbm_gbs=6000.0, write_gbs=4000.0)
    # write-bound: 8 GB written of 10 GB -> 2 ms at 4 TB/s beats 10/6 ms
    e = bench._hbm_entry("k", 4.0, 10e9, peaks, write_bytes=8e9)
    assert abs(e["floor_ms"] - 2.0) < 1e-9 and abs(e["frac_vs_floor"] - 0.5) < 1e-9
    # copy-bound: 1 GB written of 12 GB -> 2 ms at 6 TB/s beats 0.25 ms
    e = bench._hbm_entry("k", 2.5, 12e9, peaks, write_bytes=1e9)
    assert abs(e["floor_ms"] - 2.0) < 1e-9 and abs(e["frac_vs_floor"] - 0.8) < 1e-9
    # no write bytes, or no measured write rate: no floor reported
    assert "floor_ms" not in bench._hbm_entry("k", 1.0, 1e9, peaks)
    assert "floor_ms" not in bench._hbm_entry("k", 1.0, 1e9, dict(hbm_gbs=6000.0), write_bytes=1e9)


def test_output_heavy_workloads_declare_their_writes():
    """The workloads whose bytes are mostly output carry their write bytes,
    so their roofline reports the write floor."""
    for name in ("quant", "large_m_s32", "vit_fc1"):
        wl = bench.WORKLOADS[name]
        d = {}
        if wl["kind"] == "bsr":
            import synth
            crow, _ = synth.bsr_pattern(5120 // 64, 1280 // 64, 0.10, 3)
            d = dict(M=65792, K=1280, N=5120, crow=crow)
        _, dom = bench.step_accounting(wl, d)
        assert 0 < dom["write_bytes"] < dom["bytes"]


def test_profile_summaries_give_their_command():
    """Every ncu summary under profiles/ states the command that made it, with
    the clocks left alone, and runs committed files only (bench.py)."""
    pdir = os.path.join(ROOT, "profiles")
    names = sorted(f for f in os.listdir(pdir) if f.endswith(".md"))
    assert names
    for f in names:
        with open(os.path.join(pdir, f), encoding="utf-8") as fh:
            text = fh.read()
        assert "ncu " in text and "--clock-control none" in text, f
        assert "bench.py" in text, f
        assert "_work/" not in text, f

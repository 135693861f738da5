#!/usr/bin/env python
"""Benchmark of the int8 dynamic-quantization linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llm|llm_fp8|tiny|large_m|large_m_s32|vit_fc1|vit_fc2|vit_fc1_20|vit_fc2_20|
                                vit_fc1_b32|vit_fc1_b16|vit_fc1_dense|vit_fc2_dense|quant|small_m1|
                                small_m16|small_m128|mma_peak]

One step = one pass of the layer over one batch: per-token quantization of
the bf16 activations (dq_quantize_rows) and the fused i8i8->bf16 GEMM
(dq_int8_linear / dq_bsr_int8_linear).  The default workload is the
LLM-shaped dense linear: M=2048 tokens, K=4096, N=4096, 1% outlier channels.

Timing: W warm-up steps, then EXACTLY K steps captured in one CUDA graph and
replayed once, bracketed by a barrier and a device synchronize (the value).
Each kernel's average duration (kernels_ms, roofline) comes from a graph of K
launches of that kernel alone on the same buffers, timed right after.
Inputs rotate over enough copies to exceed the 126 MB L2 (config.l2).  e2e
repeats the K steps through the public API from pinned host memory, each
step's host->device copy and device->host read inside the timed region,
pipelined on three streams.  Multi-GPU: one process per GPU, token
batches sharded across ranks (weak scaling, no data-path collective); the
reported time is the max over ranks.

--impl reference times the CPU oracle (the plain C implementation the tests
use) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "int8 dyn-quant linear TOPS (dense & BSR) vs INT8 peak; quant kernel HBM GB/s"
L2_BYTES = 126 * 1024 * 1024
INT8_PER_BF16 = 2.0   # nominal dense int8 / bf16 tensor ratio (4.5 / 2.25 PFLOP/s)
METRIC_HQQ = "int4 weight-only (HQQ) linear TFLOP/s, dequant fused into the bf16 GEMM"
# The fused int4 kernel's published times at N = K = 4096, group 128, bf16
# ("Fused HQQ Quantization Gemm", pytorch/ao PR 153, the H100 results table,
# Triton column): ms by token count M.  Another machine's numbers: context.
HQQ_PAGE_H100_MS = {16: 0.1678, 32: 0.1567, 128: 0.1607, 256: 0.1515, 512: 0.1477, 1024: 0.1585}


# The CUDA sources each C-ABI entry point's kernels are compiled from (with
# the headers they include).  A stored ncu traffic figure applies only while
# these files are unchanged.
_GEMM_SOURCES = ("gemm.cu", "gemm2sm.cu", "gemm_common.cuh", "sm100.cuh", "host.cu", "internal.h")
KERNEL_SOURCES = {
    "dq_quantize_rows": ("quantize.cu", "sm100.cuh", "host.cu", "internal.h"),
    "dq_quantize_rows_fp8": ("quantize.cu", "sm100.cuh", "host.cu", "internal.h"),
    "dq_int8_linear": _GEMM_SOURCES,
    "dq_bsr_int8_linear": _GEMM_SOURCES,
    "dq_fp8_linear": _GEMM_SOURCES,
    "dq_hqq_linear": ("hqq.cu", "pipeline.cuh", "sm100.cuh", "host.cu", "internal.h"),
    "dq_s24_int8_linear": ("sparse24.cu", "pipeline.cuh", "sm100.cuh", "host.cu", "internal.h"),
    "dq_hqq_linear_t": ("hqq.cu", "pipeline.cuh", "sm100.cuh", "host.cu", "internal.h"),
}


def _strip_comments(text: str) -> str:
    """C/C++ source without its comments (string literals in these sources
    hold no comment markers) and with every run of whitespace made one space,
    so that an edit of comments or layout keeps the hash."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return re.sub(r"\s+", " ", text).strip()


def kernel_source_hash(kernel: str) -> str:
    """Hash of the CUDA sources `kernel` is built from, comments removed: a
    stored ncu traffic figure only applies to the code it was measured on."""
    import hashlib
    d = os.path.join(ROOT, "quantized_gemm_token_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + _strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def measured_traffic(workload: str, kernel: str):
    """DRAM bytes per launch (read + write) of `kernel` in `workload` from
    profiles/traffic.json (written from an ncu capture), or None when absent
    or taken on different kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            t = json.load(f)
        e = t[workload][kernel]
        return e["bytes_per_launch"] if e.get("source_hash") == kernel_source_hash(kernel) else None
    except Exception:
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


# ----------------------------------------------------------------------------
# Workloads: shapes, ops and algorithmic bytes per step.
# ----------------------------------------------------------------------------

WORKLOADS = {
    "llm": dict(kind="dense", M=2048, K=4096, N=4096, desc="LLM-shaped dense linear M=2048 K=4096 N=4096, "
                "1% x20 outlier channels, per-token quant + fused i8i8->bf16, no bias"),
    "tiny": dict(kind="dense", M=64, K=256, N=256, bias=True, desc="tiny dense linear M=64 K=256 N=256 + bias"),
    "llm_fp8": dict(kind="dense_fp8", M=2048, K=4096, N=4096,
                    desc="LLM-shaped dense linear M=2048 K=4096 N=4096, 1% x20 outlier channels, "
                         "per-token dynamic FP8 (e4m3) quant + fused e4m3 x e4m3 -> bf16 (fp32 accumulate)"),
    "large_m": dict(kind="gemm", M=38400, K=1024, N=4096, out="bf16",
                    desc="large-M int8 GEMM M=38400 K=1024 N=4096, fused bf16 epilogue"),
    "large_m_s32": dict(kind="gemm", M=38400, K=1024, N=4096, out="s32",
                        desc="large-M int8 GEMM M=38400 K=1024 N=4096, raw int32 out"),
    "vit_fc1": dict(kind="bsr", layer="fc1", desc="ViT-H fc1 BSR 10% of 64x64 blocks, M=65792 K=1280 N=5120"),
    "vit_fc2": dict(kind="bsr", layer="fc2", desc="ViT-H fc2 BSR 10% of 64x64 blocks, M=65792 K=5120 N=1280"),
    "vit_fc1_20": dict(kind="bsr", layer="fc1", keep=0.2,
                       desc="ViT-H fc1 BSR 20% of 64x64 blocks (sparsity 0.8), M=65792 K=1280 N=5120"),
    "vit_fc2_20": dict(kind="bsr", layer="fc2", keep=0.2,
                       desc="ViT-H fc2 BSR 20% of 64x64 blocks (sparsity 0.8), M=65792 K=5120 N=1280"),
    "vit_fc1_b32": dict(kind="bsr", layer="fc1", bs=32,
                        desc="ViT-H fc1 BSR 10% of 32x32 blocks, M=65792 K=1280 N=5120"),
    "vit_fc1_b16": dict(kind="bsr", layer="fc1", bs=16,
                        desc="ViT-H fc1 BSR 10% of 16x16 blocks, M=65792 K=1280 N=5120"),
    "vit_fc1_dense": dict(kind="bsr_dense", layer="fc1", desc="ViT-H fc1 dense int8 twin M=65792 K=1280 N=5120"),
    "vit_fc2_dense": dict(kind="bsr_dense", layer="fc2", desc="ViT-H fc2 dense int8 twin M=65792 K=5120 N=1280"),
    "quant": dict(kind="quant", M=16384, K=8192, desc="standalone per-token quantize X bf16 [16384, 8192]"),
    "hqq_m16": dict(kind="hqq", M=16, N=4096, K=4096, group=128,
                    desc="weight-only int4 (HQQ u4, group 128) linear M=16 N=4096 K=4096, dequant fused into a bf16 GEMM"),
    "hqq_m32": dict(kind="hqq", M=32, N=4096, K=4096, group=128,
                    desc="weight-only int4 (HQQ u4, group 128) linear M=32 N=4096 K=4096, dequant fused into a bf16 GEMM"),
    "hqq_m128": dict(kind="hqq", M=128, N=4096, K=4096, group=128,
                    desc="weight-only int4 (HQQ u4, group 128) linear M=128 N=4096 K=4096, dequant fused into a bf16 GEMM"),
    "hqq_m256": dict(kind="hqq", M=256, N=4096, K=4096, group=128,
                    desc="weight-only int4 (HQQ u4, group 128) linear M=256 N=4096 K=4096, dequant fused into a bf16 GEMM"),
    "hqq_m512": dict(kind="hqq", M=512, N=4096, K=4096, group=128,
                    desc="weight-only int4 (HQQ u4, group 128) linear M=512 N=4096 K=4096, dequant fused into a bf16 GEMM"),
    "hqq_m1024": dict(kind="hqq", M=1024, N=4096, K=4096, group=128,
                    desc="weight-only int4 (HQQ u4, group 128) linear M=1024 N=4096 K=4096, dequant fused into a bf16 GEMM"),
    "s24_llm": dict(kind="s24", M=2048, K=4096, N=4096,
                    desc="2:4-sparse int8 linear M=2048 K=4096 N=4096 (per-token quant + compressed-weight GEMM, fused bf16 epilogue)"),
    "s24_small_m16": dict(kind="s24", M=16, K=8192, N=28672,
                          desc="2:4-sparse int8 linear M=16 K=8192 N=28672 (weight stream, compressed)"),
    "hqq_t_m1024": dict(kind="hqq", M=1024, N=4096, K=4096, group=128, transposed=True,
                        desc="transposed int4 (HQQ u4, group 128) product M=1024 N=4096 K=4096 (input gradient)"),
    "small_m1": dict(kind="dense", M=1, K=8192, N=28672, desc="small-M dense linear M=1 K=8192 N=28672"),
    "small_m16": dict(kind="dense", M=16, K=8192, N=28672, desc="small-M dense linear M=16 K=8192 N=28672"),
    "small_m128": dict(kind="dense", M=128, K=8192, N=28672, desc="small-M dense linear M=128 K=8192 N=28672"),
    "mma_peak": dict(kind="mma_peak", desc="tcgen05.mma.kind::i8 128x256x32 issue loop, no HBM traffic"),
}


def _synth_inputs(name, wl, seed):
    import synth
    k = wl["kind"]
    if k == "dense_fp8":
        return synth.llm(seed)
    if k == "dense":
        if name == "llm":
            d = synth.llm(seed)
        elif name == "tiny":
            d = synth.tiny(seed)
        else:
            d = synth.small_m(seed, M=wl["M"], K=wl["K"], N=wl["N"])
        return d
    if k == "gemm":
        return synth.large_m(seed)
    if k in ("bsr", "bsr_dense"):
        return synth.vit_h_bsr(seed, wl["layer"], keep=wl.get("keep", 0.10), bs=wl.get("bs", 64))
    if k == "quant":
        return synth.quant_sweep(seed)
    if k == "s24":
        return synth.s24(seed, M=wl["M"], K=wl["K"], N=wl["N"])
    if k == "hqq":
        d = synth.hqq(seed, M=wl["M"], N=wl["N"], K=wl["K"], group=wl["group"])
        if wl.get("transposed"):
            d["x"] = synth.normal_bf16((wl["M"], wl["N"]), 1.0, seed)
        return d
    return {}


def step_accounting(wl, d):
    """(ops per step, dominant kernel name, its algorithmic units)."""
    k = wl["kind"]
    if k in ("dense", "gemm", "dense_fp8"):
        M, K, N = wl["M"], wl["K"], wl["N"]
        ops = 2.0 * M * N * K
        out_b = 4 if wl.get("out") == "s32" else 2
        gemm_bytes = M * K + N * K + M * N * out_b + 4 * (M + N)
        return ops, dict(kernel="dq_fp8_linear" if k == "dense_fp8" else "dq_int8_linear", ops=ops,
                         bytes=gemm_bytes, quant_bytes=(3 * M * K + 4 * M) if k != "gemm" else 0,
                         write_bytes=M * N * out_b)
    if k in ("bsr", "bsr_dense"):
        M, K, N = d["M"], d["K"], d["N"]
        nnzb = int(d["crow"][-1])
        bs = wl.get("bs", 64)
        ops = 2.0 * M * nnzb * bs * bs if k == "bsr" else 2.0 * M * N * K
        wbytes = nnzb * bs * bs if k == "bsr" else N * K
        return ops, dict(kernel="dq_bsr_int8_linear" if k == "bsr" else "dq_int8_linear", ops=ops,
                         bytes=M * K + wbytes + 2 * M * N + 4 * (M + N), quant_bytes=3 * M * K + 4 * M,
                         write_bytes=2 * M * N)
    if k == "quant":
        M, K = wl["M"], wl["K"]
        return 0.0, dict(kernel="dq_quantize_rows", ops=0.0, bytes=3 * M * K + 4 * M, quant_bytes=3 * M * K + 4 * M,
                         write_bytes=M * K + 4 * M)
    if k == "s24":
        M, K, N = wl["M"], wl["K"], wl["N"]
        ops = 2.0 * M * N * K          # dense-equivalent work of the 2:4 product
        gemm_bytes = M * K + N * K // 2 + N * K // 8 + 2 * M * N + 4 * (M + N)
        return ops, dict(kernel="dq_s24_int8_linear", ops=ops, bytes=gemm_bytes, quant_bytes=3 * M * K + 4 * M)
    if k == "hqq":
        M, K, N = wl["M"], wl["K"], wl["N"]
        ops = 2.0 * M * N * K
        n_in, n_out = (N, K) if wl.get("transposed") else (K, N)
        # activations + packed codes + bf16 scale and zero per group + bf16 output
        b = 2 * M * n_in + N * K // 2 + 2 * 2 * N * (K // wl["group"]) + 2 * M * n_out
        return ops, dict(kernel="dq_hqq_linear_t" if wl.get("transposed") else "dq_hqq_linear", ops=ops, bytes=b,
                         quant_bytes=0)
    return 0.0, {}


# ----------------------------------------------------------------------------
# Clock sampling during the timed region (NVML reads only).
# ----------------------------------------------------------------------------

class ClockSampler:
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = None
            try:
                from cuda.bindings import runtime as rt
                err, bus = rt.cudaDeviceGetPCIBusId(64, device_index)
                if err == rt.cudaError_t.cudaSuccess:
                    bus = bus.split(b"\x00")[0] if isinstance(bus, bytes) else str(bus).encode()
                    self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = None
            if self._h is None:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def _to_dev(torch, a):
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _to_dev_bf16(torch, bits):
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _finish(st):
    """One step = the workload's kernels in order, each one launch."""
    kernels = st["kernels"]

    def step(c, stream):
        for k in kernels:
            k(c, stream)
    st["step"], st["n_kernels"] = step, len(kernels)
    return st


def make_state(name, wl, dq, torch, seed):
    import numpy as np
    k = wl["kind"]
    d = _synth_inputs(name, wl, seed)
    st = dict(d=d, kernels=[])
    if k == "mma_peak":
        return st
    if k == "quant":
        x = _to_dev_bf16(torch, d["x"])
        M, K = x.shape
        st["copies"] = [dict(x=x if i == 0 else x.clone()) for i in range(_ncopies(x.numel() * 3))]
        q = torch.empty((M, K), dtype=torch.int8, device="cuda")
        s = torch.empty((M,), dtype=torch.float32, device="cuda")
        st["q"], st["s"] = q, s
        st["h2d"] = [("x", x.numel() * 2)]
        st["d2h"] = [("q", M * K), ("s", M * 4)]

        st["kernels"] = [lambda c, stream: dq.dq_quantize_rows(c["x"], q, s, stream=stream)]
        st["names"] = ["dq_quantize_rows"]
        return _finish(st)
    if k == "gemm":
        A, B = _to_dev(torch, d["a"]), _to_dev(torch, d["b"])
        sr, sc = _to_dev(torch, d["s_row"]), _to_dev(torch, d["s_col"])
        M, K = A.shape
        N = B.shape[0]
        out_s32 = wl["out"] == "s32"
        out = torch.empty((M, N), dtype=torch.int32 if out_s32 else torch.bfloat16, device="cuda")
        n = _ncopies(A.numel() + B.numel())
        st["copies"] = [dict(A=A if i == 0 else A.clone(), B=B if i == 0 else B.clone()) for i in range(n)]
        st["h2d"] = [("A", M * K)]
        st["d2h"] = [("out", out.numel() * out.element_size())]

        st["kernels"] = [lambda c, stream: dq.dq_int8_linear(c["A"], sr, c["B"], sc, out=out,
                                                             out_dtype="s32" if out_s32 else "bf16", stream=stream)]
        st["names"] = ["dq_int8_linear"]
        st["out"] = out
        return _finish(st)
    # layer workloads: quantize + GEMM
    if k == "dense_fp8":
        w = _to_dev(torch, d["w"])
        wq, sc = dq.dq_quantize_weight_fp8(w)
        del w
        M, K, N = d["x"].shape[0], d["x"].shape[1], d["w"].shape[0]
        x = _to_dev_bf16(torch, d["x"])
        n = _ncopies(x.numel() * 2 + wq.numel())
        st["copies"] = [dict(x=x if i == 0 else x.clone(), W=wq if i == 0 else wq.clone()) for i in range(n)]
        q = torch.empty((M, K), dtype=torch.uint8, device="cuda")
        s = torch.empty((M,), dtype=torch.float32, device="cuda")
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        st.update(q=q, s=s, out=out)
        st["h2d"] = [("x", M * K * 2)]
        st["d2h"] = [("out", M * N * 2)]

        st["kernels"] = [
            lambda c, stream: dq.dq_quantize_rows_fp8(c["x"], q, s, stream=stream),
            lambda c, stream: dq.dq_fp8_linear(q, s, c["W"], sc, out=out, stream=stream)]
        st["names"] = ["dq_quantize_rows_fp8", "dq_fp8_linear"]
        return _finish(st)
    if k == "dense":
        w = _to_dev(torch, d["w"])
        wq, sc = dq.dq_quantize_weight(w)
        del w
        M, K, N = d["x"].shape[0], d["x"].shape[1], d["w"].shape[0]
        bias = _to_dev_bf16(torch, d["bias"]) if d.get("bias") is not None else None
        x = _to_dev_bf16(torch, d["x"])
        n = _ncopies(x.numel() * 2 + wq.numel())
        st["copies"] = [dict(x=x if i == 0 else x.clone(), W=wq if i == 0 else wq.clone()) for i in range(n)]
        q = torch.empty((M, K), dtype=torch.int8, device="cuda")
        s = torch.empty((M,), dtype=torch.float32, device="cuda")
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        nws = dq.dq_int8_linear_workspace_size(M, N, K)
        ws = torch.zeros(nws, dtype=torch.uint8, device="cuda") if nws else None
        st.update(q=q, s=s, out=out, ws=ws)
        st["h2d"] = [("x", M * K * 2)]
        st["d2h"] = [("out", M * N * 2)]

        st["kernels"] = [
            lambda c, stream: dq.dq_quantize_rows(c["x"], q, s, stream=stream),
            lambda c, stream: dq.dq_int8_linear(q, s, c["W"], sc, bias=bias, out=out, workspace=ws, stream=stream)]
        st["names"] = ["dq_quantize_rows", "dq_int8_linear"]
        return _finish(st)
    if k == "s24":
        w = _to_dev(torch, d["w"])
        wq, sc = dq.dq_quantize_weight(w)
        del w
        vals, meta = dq.dq_s24_compress(wq)
        del wq
        M, K, N = wl["M"], wl["K"], wl["N"]
        x = _to_dev_bf16(torch, d["x"])
        n = _ncopies(x.numel() * 2 + vals.numel() + meta.numel())
        st["copies"] = [dict(x=x if i == 0 else x.clone(), V=vals if i == 0 else vals.clone(),
                             Mt=meta if i == 0 else meta.clone()) for i in range(n)]
        q = torch.empty((M, K), dtype=torch.int8, device="cuda")
        s = torch.empty((M,), dtype=torch.float32, device="cuda")
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        nws = dq.dq_s24_workspace_size(M, N, K)
        ws = torch.zeros(nws, dtype=torch.uint8, device="cuda") if nws else None
        st.update(q=q, s=s, out=out, ws=ws)
        st["h2d"] = [("x", M * K * 2)]
        st["d2h"] = [("out", M * N * 2)]
        st["kernels"] = [
            lambda c, stream: dq.dq_quantize_rows(c["x"], q, s, stream=stream),
            lambda c, stream: dq.dq_s24_int8_linear(q, s, c["V"], c["Mt"], sc, out=out, workspace=ws, stream=stream)]
        st["names"] = ["dq_quantize_rows", "dq_s24_int8_linear"]
        return _finish(st)
    if k == "hqq":
        trans = bool(wl.get("transposed"))
        M, K, N, group = wl["M"], wl["K"], wl["N"], wl["group"]
        packed = dq.dq_hqq_pack(_to_dev(torch, d["codes"]))
        sc = dq.dq_hqq_group_major(_to_dev_bf16(torch, d["scale"]))
        ze = dq.dq_hqq_group_major(_to_dev_bf16(torch, d["zero"]))
        x = _to_dev_bf16(torch, d["x"])
        n = _ncopies(x.numel() * 2 + packed.numel() + 2 * sc.numel() * 2)
        st["copies"] = [dict(x=x if i == 0 else x.clone(), P=packed if i == 0 else packed.clone(),
                             S=sc if i == 0 else sc.clone(), Z=ze if i == 0 else ze.clone()) for i in range(n)]
        n_out = K if trans else N
        out = torch.empty((M, n_out), dtype=torch.bfloat16, device="cuda")
        nws = dq.dq_hqq_workspace_size(M, N, K, trans)
        ws = torch.zeros(nws, dtype=torch.uint8, device="cuda") if nws else None
        st.update(out=out, ws=ws)
        st["h2d"] = [("x", x.numel() * 2)]
        st["d2h"] = [("out", M * n_out * 2)]
        fn = dq.dq_hqq_linear_t if trans else dq.dq_hqq_linear
        st["kernels"] = [lambda c, stream: fn(c["x"], c["P"], c["S"], c["Z"], group, out=out, workspace=ws,
                                             stream=stream)]
        st["names"] = ["dq_hqq_linear_t" if trans else "dq_hqq_linear"]
        return _finish(st)
    if k in ("bsr", "bsr_dense"):
        w = _to_dev(torch, d["w"])
        wq, sc = dq.dq_quantize_weight(w)
        del w
        crow, col = _to_dev(torch, d["crow"]), _to_dev(torch, d["col"])
        values = dq.dq_bsr_pack(wq, crow, col, block=wl.get("bs", 64))
        M, K, N = d["M"], d["K"], d["N"]
        x = _to_dev_bf16(torch, d["x"])
        del d["x"]
        n = _ncopies(x.numel() * 2)
        st["copies"] = [dict(x=x if i == 0 else x.clone()) for i in range(n)]
        q = torch.empty((M, K), dtype=torch.int8, device="cuda")
        s = torch.empty((M,), dtype=torch.float32, device="cuda")
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        st.update(q=q, s=s, out=out)
        st["h2d"] = [("x", M * K * 2)]
        st["d2h"] = [("out", M * N * 2)]
        dense = k == "bsr_dense"

        def gemm(c, stream):
            if dense:
                dq.dq_int8_linear(q, s, wq, sc, out=out, stream=stream)
            else:
                dq.dq_bsr_int8_linear(q, s, N, crow, col, values, sc, out=out, stream=stream)
        st["kernels"] = [lambda c, stream: dq.dq_quantize_rows(c["x"], q, s, stream=stream), gemm]
        st["names"] = ["dq_quantize_rows", "dq_int8_linear" if dense else "dq_bsr_int8_linear"]
        return _finish(st)
    raise ValueError(k)


def _ncopies(bytes_per_copy):
    n = 1
    while n * bytes_per_copy <= 2 * L2_BYTES and n < 64:
        n += 1
    return n


def run_gpu(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    import quantized_gemm_token_b200 as dq

    torch.cuda.set_device(local_rank)
    dev_index = local_rank
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180),
                                device_id=torch.device("cuda", local_rank))
    name = args.workload
    wl = WORKLOADS[name]
    peaks = load_peaks()
    torch.manual_seed(0)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    stream = torch.cuda.current_stream()

    if wl["kind"] == "mma_peak":
        iters = 20000
        for _ in range(max(args.warmup, 3)):
            dq.dq_mma_peak_probe(0, iters)
        torch.cuda.synchronize()
        sms = torch.cuda.get_device_properties(local_rank).multi_processor_count
        st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev_index) as cs:
            st.record()
            for _ in range(args.steps):
                dq.dq_mma_peak_probe(0, iters)
            en.record()
            torch.cuda.synchronize()
        ms = st.elapsed_time(en)
        assert dq.dq_sync_status() == dq.DQ_OK
        tops = args.steps * sms * iters * 2.0 * 128 * 256 * 32 / (ms * 1e-3) / 1e12
        line = dict(metric="int8 tcgen05.mma issue-rate peak", value=round(tops, 1), unit="TOPS", n_gpus=world,
                    steps=args.steps, warmup=args.warmup, ms_per_step=round(ms / args.steps, 4),
                    higher_is_better=True, scaling="weak", vs_baseline=None, dtype="int8", data="synthetic",
                    config=dict(workload=wl["desc"], sms=sms, mma_per_cta=iters), clocks=cs.summary(),
                    gpu_launches=args.steps)
        if rank == 0:
            print(json.dumps(line), flush=True)
        return

    # seed per rank: each rank holds its own token batch (weak scaling)
    state = make_state(name, wl, dq, torch, seed=rank)
    ops, dom = step_accounting(wl, state["d"])
    copies = state["copies"]
    step = state["step"]
    nk = state["n_kernels"]
    K = args.steps

    # warm-up (also first-call set-up: tensor-map encoder, kernel attributes)
    for i in range(max(args.warmup, 3)):
        step(copies[i % len(copies)], stream)
    torch.cuda.synchronize()
    assert dq.dq_sync_status() == dq.DQ_OK

    def capture(launch):
        """A CUDA graph of K launches of `launch(i, stream)`, uploaded once."""
        graph = torch.cuda.CUDAGraph()
        cap_stream = torch.cuda.Stream()
        cap_stream.wait_stream(stream)
        with torch.cuda.stream(cap_stream):
            graph.capture_begin()
            for i in range(K):
                launch(i, cap_stream)
            graph.capture_end()
        stream.wait_stream(cap_stream)
        graph.replay()            # one untimed replay (graph upload)
        torch.cuda.synchronize()
        return graph

    def timed_replay(graph):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        graph.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    # The timed region: one graph of exactly K steps (nothing between kernels).
    graph = capture(lambda i, cs: step(copies[i % len(copies)], cs))
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev_index) as cs:
        start.record()
        graph.replay()
        end.record()
        torch.cuda.synchronize()
    barrier()
    total_ms = start.elapsed_time(end)
    assert dq.dq_sync_status() == dq.DQ_OK
    del graph
    # Per-kernel durations: right after, a graph of K launches of each kernel
    # alone (same buffers, same input rotation), timed with events around it.
    per_kernel_ms = []
    for j, kern in enumerate(state["kernels"]):
        gj = capture(lambda i, cs, kern=kern: kern(copies[i % len(copies)], cs))
        per_kernel_ms.append(timed_replay(gj) / K)
        del gj
    assert dq.dq_sync_status() == dq.DQ_OK
    total_ms_max = max_over_ranks(total_ms)

    value = ops * world * K / (total_ms_max * 1e-3) / 1e12 if ops else None
    unit = "TOPS"
    if wl["kind"] == "quant":
        value = dom["bytes"] * world * K / (total_ms_max * 1e-3) / 1e9
        unit = "GB/s"

    # roofline of the dominant kernel
    j = state["names"].index(dom["kernel"])
    avg_ms = per_kernel_ms[j]
    int8_peak = peaks["bf16"] * INT8_PER_BF16
    if dom["kernel"] == "dq_quantize_rows" or wl.get("out") == "s32" or wl["kind"] == "bsr":
        t_tensor = dom["ops"] / (int8_peak * 1e12) if dom["ops"] else 0.0
        t_hbm = dom["bytes"] / (peaks["hbm_gbs"] * 1e9)
        hbm_bound = t_hbm >= t_tensor
    else:
        hbm_bound = False
    if dom["kernel"].startswith("dq_int8_linear") and wl["kind"] == "dense" and wl["M"] <= 128:
        hbm_bound = True     # small-M: weight streaming
    if wl["kind"] == "s24":
        hbm_bound = dom["bytes"] / (peaks["hbm_gbs"] * 1e9) >= dom["ops"] / (int8_peak * 1e12)
    hqq = wl["kind"] == "hqq"
    if hqq:
        int8_peak = peaks["bf16"]      # bf16 operands on the tensor cores
        hbm_bound = dom["bytes"] / (peaks["hbm_gbs"] * 1e9) >= dom["ops"] / (int8_peak * 1e12)
    if hbm_bound:
        achieved = dom["bytes"] / (avg_ms * 1e-3) / 1e9
        roof = dict(bound="hbm", achieved=round(achieved, 1), peak=peaks["hbm_gbs"], unit="GB/s",
                    frac=round(achieved / peaks["hbm_gbs"], 4), traffic=None,
                    peak_source=f"{peaks['src']} HBM copy bandwidth")
    else:
        achieved = dom["ops"] / (avg_ms * 1e-3) / 1e12
        roof = dict(bound="tensor", achieved=round(achieved, 1), peak=round(int8_peak, 1), unit="TOPS",
                    frac=round(achieved / int8_peak, 4), traffic=None,
                    peak_source=f"{peaks['src']} bf16 burst x {INT8_PER_BF16:g} (nominal int8/bf16 ratio)")
        if hqq:
            roof.update(unit="TFLOP/s", peak_source=f"{peaks['src']} bf16 burst (cuBLAS bf16 GEMM)")
    probe = None
    if world == 1 and not args.no_secondary:
        probe = probe_int8_tops(dq, torch)
    if world == 1 and (hbm_bound or not args.no_secondary):
        peaks["write_gbs"] = probe_hbm_write_gbs(torch)
    if hbm_bound and dom.get("write_bytes") and peaks.get("write_gbs"):
        # floor: the output at the measured write-only rate, or all bytes at
        # the copy rate, whichever is longer
        floor_ms = max(dom["write_bytes"] / (peaks["write_gbs"] * 1e9), dom["bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e3
        roof["write_floor"] = dict(write_gbs=round(peaks["write_gbs"], 1), write_bytes=int(dom["write_bytes"]),
                                   floor_ms=round(floor_ms, 5), frac_vs_floor=round(floor_ms / avg_ms, 4),
                                   source="torch fill of a 1 GiB buffer, timed in this run")
    if not hbm_bound and probe is not None and not hqq:
        roof["frac_vs_probe"] = round(achieved / probe, 4)
        roof["probe_tops"] = round(probe, 1)
        roof["frac_vs_spec"] = round(achieved / SPEC_INT8_TOPS, 4)
    elif hbm_bound:
        roof["frac_vs_spec"] = round(achieved / SPEC_HBM_GBS, 4)
    roof["kernel"] = dom["kernel"]
    roof["traffic"] = measured_traffic(name, dom["kernel"])
    roof["avg_launch_ms"] = round(avg_ms, 5)
    roof["algorithmic_bytes" if hbm_bound else "algorithmic_ops"] = dom["bytes"] if hbm_bound else dom["ops"]
    kernels_ms = {n: round(per_kernel_ms[i], 5) for i, n in enumerate(state["names"])}

    # end to end through the public API with host buffers
    e2e = None
    if wl["kind"] in ("dense", "bsr", "bsr_dense", "quant", "gemm", "dense_fp8", "hqq", "s24"):
        e2e = run_e2e(args, wl, state, dq, torch, stream, ops, dom, world, max_over_ranks)

    vs_baseline = None
    dtype = "e4m3" if wl["kind"] == "dense_fp8" else "int8"
    metric = METRIC
    if hqq:
        unit, metric, dtype = "TFLOP/s", METRIC_HQQ, "bf16"
        page_ms = HQQ_PAGE_H100_MS.get(wl["M"]) if not wl.get("transposed") else None
        if page_ms:
            vs_baseline = round(value / (ops / (page_ms * 1e-3) / 1e12), 2)
    line = dict(metric=metric, value=round(value, 2) if value is not None else None, unit=unit, n_gpus=world,
                steps=K, warmup=args.warmup, ms_per_step=round(total_ms_max / K, 5), higher_is_better=True,
                scaling="weak", vs_baseline=vs_baseline, dtype=dtype,
                data="synthetic",
                config=dict(workload=wl["desc"], tokens_per_rank=state["d"].get("M", wl.get("M")),
                            parallelism=f"dp{world} (token rows sharded, weights replicated, no collective)",
                            l2=f"inputs rotate over {len(copies)} copies (> 2x the 126 MB L2)",
                            timing="value: one CUDA graph of the K steps, events around it; "
                                   "kernels_ms / roofline: per kernel, a graph of K launches of that "
                                   "kernel alone on the same buffers, events around it; e2e: K steps "
                                   "through the public API, each with its pinned-host H2D copy and D2H "
                                   "read, pipelined on three streams (copy-in / kernels / copy-out)",
                            kernels_ms=kernels_ms),
                roofline=roof, e2e=e2e, gpu_launches=nk * K, clocks=cs.summary())
    if wl["kind"] in ("dense", "bsr", "bsr_dense", "s24"):
        line["config"]["weight_prep"] = ("weights quantized per channel on the GPU by dq_quantize_weight, "
                                         "whose codes and scales the parity tests check bit for bit against "
                                         "the oracle's routine")
    if hqq:
        line["config"]["weight"] = (f"int4 {'s4' if wl.get('signed') else 'u4'} codes, group {wl['group']}, "
                                    "bf16 scales and zero points; dequantized in the GEMM")
    if probe is not None:
        line["probes"] = dict(int8_mma_tops=round(probe, 1), hbm_write_gbs=round(peaks["write_gbs"], 1))
    if probe is not None and name == "llm":
        line["secondary"] = secondary_measurements(dq, torch, peaks, probe, K)
        line["secondary"]["_about"] = (
            "the metric's other workloads, timed in this run on 1 GPU: each kernel as a graph of K launches "
            "(events around it), inputs drawn on the device with the parity workloads' shapes and "
            "distributions; frac = achieved / measured peak (HBM copy, or bf16 burst x 2 for int8), "
            "frac_vs_probe = / the int8 tcgen05.mma issue rate measured by dq_mma_peak_probe in this run, "
            "frac_vs_spec = / the nominal 4.5 POPS or 8 TB/s")
    if wl["kind"] == "s24":
        line["config"]["weight"] = "2:4 sparse int8, compressed (two values + a position nibble per group of four)"
    if rank == 0 and world == 1 and not args.no_cpu_baseline and wl["kind"] in ("dense", "bsr", "quant", "gemm",
                                                                                 "hqq", "s24"):
        line["cpu_baseline"] = cpu_baseline(name, wl, state["d"], budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ----------------------------------------------------------------------------
# The metric's other halves, measured in the same run (1 GPU): the BSR layer
# against its dense twin, the standalone quantize, the few-token weight
# stream, the large-M GEMM, and the tensor-pipe issue-rate probe.
# ----------------------------------------------------------------------------

SPEC_INT8_TOPS = 4500.0   # B200 dense int8, nominal
SPEC_HBM_GBS = 8000.0     # B200 HBM3e, nominal


def _graph_ms(torch, launch, n):
    """Average device time of `launch(i, stream)` over a CUDA graph of n
    launches (events around one replay, after an upload replay)."""
    stream = torch.cuda.current_stream()
    for i in range(3):
        launch(i, stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(stream)
    with torch.cuda.stream(cs):
        graph.capture_begin()
        for i in range(n):
            launch(i, cs)
        graph.capture_end()
    stream.wait_stream(cs)
    graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    graph.replay()
    b.record()
    mhz = _sm_clock_mhz()       # read while the replay runs
    torch.cuda.synchronize()
    del graph
    _LAST_CLOCK[0] = mhz
    return a.elapsed_time(b) / n


_LAST_CLOCK = [None]
_NVML = {}


def _sm_clock_mhz():
    """SM clock of the current device through NVML (None if unavailable)."""
    try:
        if "h" not in _NVML:
            import pynvml
            pynvml.nvmlInit()
            _NVML["nv"] = pynvml
            _NVML["h"] = pynvml.nvmlDeviceGetHandleByIndex(int(os.environ.get("LOCAL_RANK", "0")))
        return _NVML["nv"].nvmlDeviceGetClockInfo(_NVML["h"], _NVML["nv"].NVML_CLOCK_SM)
    except Exception:
        return None


def probe_int8_tops(dq, torch, iters=20000, reps=5):
    """The tcgen05.mma.kind::i8 issue rate (dq_mma_peak_probe: one CTA per SM,
    128x256x32 MMAs from resident shared-memory tiles)."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    for _ in range(2):
        dq.dq_mma_peak_probe(0, iters)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        dq.dq_mma_peak_probe(0, iters)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    return sms * iters * 2.0 * 128 * 256 * 32 / (ms * 1e-3) / 1e12


def probe_hbm_write_gbs(torch, nbytes=1 << 30, reps=10):
    """Write-only HBM bandwidth: torch's fill of a 1 GiB buffer (a plain
    vectorized store stream), timed with events.  On this part a pure write
    stream runs well below the copy bandwidth, so kernels whose bytes are
    mostly output are also reported against the floor it sets."""
    x = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        x.fill_(1)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        x.fill_(1)
    b.record()
    torch.cuda.synchronize()
    gbs = nbytes * reps / (a.elapsed_time(b) * 1e-3) / 1e9
    del x
    torch.cuda.empty_cache()
    return gbs


def _tensor_entry(name, ms, ops, peaks, probe):
    int8_peak = peaks["bf16"] * INT8_PER_BF16
    tops = ops / (ms * 1e-3) / 1e12
    return dict(kernel=name, kernel_ms=round(ms, 5), bound="tensor", achieved=round(tops, 1), unit="TOPS",
                peak=round(int8_peak, 1), frac=round(tops / int8_peak, 4), frac_vs_probe=round(tops / probe, 4),
                frac_vs_spec=round(tops / SPEC_INT8_TOPS, 4), sm_mhz=_LAST_CLOCK[0])


def _hbm_entry(name, ms, nbytes, peaks, write_bytes=0):
    gbs = nbytes / (ms * 1e-3) / 1e9
    e = dict(kernel=name, kernel_ms=round(ms, 5), bound="hbm", achieved=round(gbs, 1), unit="GB/s",
             peak=peaks["hbm_gbs"], frac=round(gbs / peaks["hbm_gbs"], 4), frac_vs_spec=round(gbs / SPEC_HBM_GBS, 4),
             algorithmic_bytes=int(nbytes), sm_mhz=_LAST_CLOCK[0])
    wgbs = peaks.get("write_gbs")
    if write_bytes and wgbs:
        # floor: the output at the measured write-only rate, or all bytes at
        # the copy rate, whichever is longer
        floor_ms = max(write_bytes / (wgbs * 1e9), nbytes / (peaks["hbm_gbs"] * 1e9)) * 1e3
        e.update(write_bytes=int(write_bytes), floor_ms=round(floor_ms, 5), frac_vs_floor=round(floor_ms / ms, 4))
    return e


def secondary_measurements(dq, torch, peaks, probe, n):
    """Kernel times of the metric's other workloads, each a graph of n
    launches on inputs drawn on the device (seeded; the same shapes and value
    distributions as the parity workloads).  Inputs larger than the 126 MB L2,
    or rotated over copies that are."""
    import numpy as np
    import synth
    out = {}
    gen = torch.Generator(device="cuda")

    def randn(shape, std, seed):
        gen.manual_seed(seed)
        return torch.randn(shape, generator=gen, device="cuda", dtype=torch.float32) * std

    # Each workload starts after a 1 s pause, so that every one is timed from
    # the same clock state (long runs of the large ones can leave the part
    # under its power cap for a while); each entry records the SM clock read
    # during its timed replay.
    pause = lambda: time.sleep(1.0)  # noqa: E731
    pause()
    # standalone quantize, X bf16 [16384, 8192] (268 MB read)
    M, K = 16384, 8192
    x = randn((M, K), 1.0, 11).to(torch.bfloat16)
    q = torch.empty((M, K), dtype=torch.int8, device="cuda")
    s = torch.empty((M,), dtype=torch.float32, device="cuda")
    ms = _graph_ms(torch, lambda i, st: dq.dq_quantize_rows(x, q, s, stream=st), n)
    out["quant_16384x8192"] = _hbm_entry("dq_quantize_rows", ms, 3 * M * K + 4 * M, peaks, M * K + 4 * M)
    del x, q, s

    pause()
    # few-token dense linear M=16, K=8192, N=28672: the weight stream (235 MB)
    M, K, N = 16, 8192, 28672
    wq, sc = dq.dq_quantize_weight(randn((N, K), 0.02, 12))
    x = randn((M, K), 1.0, 13).to(torch.bfloat16)
    q, s = dq.dq_quantize_rows(x)
    o = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    nws = dq.dq_int8_linear_workspace_size(M, N, K)
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda") if nws else None
    ms = _graph_ms(torch, lambda i, st: dq.dq_int8_linear(q, s, wq, sc, out=o, workspace=ws, stream=st), n)
    out["small_m16_8192x28672"] = _hbm_entry("dq_int8_linear", ms, N * K + M * K + 2 * M * N + 4 * (M + N), peaks)
    del wq, sc, x, q, s, o, ws

    pause()
    # large-M GEMM M=38400, K=1024, N=4096, bf16 out (A rotated over 4 copies)
    M, K, N = 38400, 1024, 4096
    gen.manual_seed(14)
    As = [torch.randint(-127, 128, (M, K), generator=gen, dtype=torch.int8, device="cuda") for _ in range(4)]
    B = torch.randint(-127, 128, (N, K), generator=gen, dtype=torch.int8, device="cuda")
    sr = torch.rand((M,), generator=gen, device="cuda") * 0.049 + 0.001
    scl = torch.rand((N,), generator=gen, device="cuda") * 0.049 + 0.001
    o = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ms = _graph_ms(torch, lambda i, st: dq.dq_int8_linear(As[i % 4], sr, B, scl, out=o, stream=st), n)
    out["large_m_38400x1024x4096_bf16"] = _tensor_entry("dq_int8_linear", ms, 2.0 * M * N * K, peaks, probe)
    del As, B, sr, scl, o

    # ViT-H MLP at batch 256: 10 % of the 64x64 blocks kept, BSR against the
    # dense twin (the same masked weight, dense int8) and the layer with its
    # quantize
    for layer in ("fc1", "fc2"):
        pause()
        K, N = (1280, 5120) if layer == "fc1" else (5120, 1280)
        M = 256 * 257
        crow, col = synth.bsr_pattern(N // 64, K // 64, 0.10, (0 if layer == "fc1" else 100) + 3)
        w = randn((N, K), 0.02, 15 + K)
        bmask = torch.zeros((N // 64, K // 64), dtype=torch.bool, device="cuda")
        rows = np.repeat(np.arange(N // 64), np.diff(crow))
        bmask[torch.from_numpy(rows).cuda(), torch.from_numpy(col.astype(np.int64)).cuda()] = True
        w *= bmask.repeat_interleave(64, 0).repeat_interleave(64, 1)
        wq, sc = dq.dq_quantize_weight(w)
        del w, bmask
        crow_d, col_d = torch.from_numpy(crow).cuda(), torch.from_numpy(col).cuda()
        vals = dq.dq_bsr_pack(wq, crow_d, col_d)
        x = randn((M, K), 1.0, 16 + K).to(torch.bfloat16)
        q = torch.empty((M, K), dtype=torch.int8, device="cuda")
        s = torch.empty((M,), dtype=torch.float32, device="cuda")
        o = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ms_q = _graph_ms(torch, lambda i, st: dq.dq_quantize_rows(x, q, s, stream=st), n)
        ms_b = _graph_ms(torch, lambda i, st: dq.dq_bsr_int8_linear(q, s, N, crow_d, col_d, vals, sc, out=o,
                                                                      stream=st), n)
        clk_b = _LAST_CLOCK[0]
        ms_d = _graph_ms(torch, lambda i, st: dq.dq_int8_linear(q, s, wq, sc, out=o, stream=st), n)
        nnzb = int(crow[-1])
        e = _hbm_entry("dq_bsr_int8_linear", ms_b, M * K + nnzb * 4096 + 2 * M * N + 4 * (M + N), peaks, 2 * M * N)
        e["sm_mhz"] = clk_b
        e["dense_twin"] = _tensor_entry("dq_int8_linear", ms_d, 2.0 * M * N * K, peaks, probe)
        e["quantize_ms"] = round(ms_q, 5)
        e["gemm_speedup_vs_dense"] = round(ms_d / ms_b, 3)
        e["layer_speedup_vs_dense"] = round((ms_q + ms_d) / (ms_q + ms_b), 3)
        out[f"vit_h_{layer}_bsr10_{M}x{K}x{N}"] = e
        del wq, sc, vals, x, q, s, o
    # LLM-shaped layer with a 2:4-sparse weight (the sparse tensor-core MMA)
    # and with dynamic FP8, against the dense int8 GEMM of the same shape;
    # few-token 2:4 weight stream
    for (M, K, N, tag) in ((2048, 4096, 4096, "s24_llm_2048x4096x4096"), (16, 8192, 28672, "s24_small_m16_8192x28672")):
        pause()
        w = randn((N, K), 0.02, 17 + M)
        # a uniform 2:4 mask: one of the six position pairs per group of four
        pairs = torch.tensor([[1, 1, 0, 0], [1, 0, 1, 0], [1, 0, 0, 1], [0, 1, 1, 0], [0, 1, 0, 1], [0, 0, 1, 1]],
                             dtype=torch.float32, device="cuda")
        keep = pairs[torch.randint(0, 6, (N, K // 4), generator=gen, device="cuda")]
        w = (w.view(N, K // 4, 4) * keep).view(N, K)
        del keep
        wq, sc = dq.dq_quantize_weight(w)
        del w
        vals, meta = dq.dq_s24_compress(wq)
        x = randn((M, K), 1.0, 18 + M).to(torch.bfloat16)
        q, s = dq.dq_quantize_rows(x)
        o = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        nws = dq.dq_s24_workspace_size(M, N, K)
        ws = torch.zeros(nws, dtype=torch.uint8, device="cuda") if nws else None
        ms_s = _graph_ms(torch, lambda i, st: dq.dq_s24_int8_linear(q, s, vals, meta, sc, out=o, workspace=ws, stream=st), n)
        clk_s = _LAST_CLOCK[0]
        nwd = dq.dq_int8_linear_workspace_size(M, N, K)
        wsd = torch.zeros(nwd, dtype=torch.uint8, device="cuda") if nwd else None
        ms_d = _graph_ms(torch, lambda i, st: dq.dq_int8_linear(q, s, wq, sc, out=o, workspace=wsd, stream=st), n)
        if M > 128:
            e = _tensor_entry("dq_s24_int8_linear", ms_s, 2.0 * M * N * K, peaks, probe)
            e["ops_note"] = "dense-equivalent ops (2 M N K) of the 2:4 product"
        else:
            e = _hbm_entry("dq_s24_int8_linear", ms_s, N * K // 2 + N * K // 8 + M * K + 2 * M * N + 4 * (M + N), peaks)
        e["sm_mhz"] = clk_s
        e["dense_int8_ms"] = round(ms_d, 5)
        e["speedup_vs_dense_int8"] = round(ms_d / ms_s, 3)
        out[tag] = e
        del wq, sc, vals, meta, x, q, s, o, ws, wsd
    M, K, N = 2048, 4096, 4096
    pause()
    wq8, sc8 = dq.dq_quantize_weight_fp8(randn((N, K), 0.02, 19))
    q8, s8 = dq.dq_quantize_rows_fp8(randn((M, K), 1.0, 20).to(torch.bfloat16))
    o = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ms = _graph_ms(torch, lambda i, st: dq.dq_fp8_linear(q8, s8, wq8, sc8, out=o, stream=st), n)
    e = _tensor_entry("dq_fp8_linear", ms, 2.0 * M * N * K, peaks, probe)
    e["peak_note"] = "e4m3 x e4m3 nominal rate = the int8 rate (bf16 x 2)"
    out["fp8_llm_2048x4096x4096"] = e
    del wq8, sc8, q8, s8, o
    # weight-only int4 (HQQ) at the page's few-token and 1024-token shapes
    N = K = 4096
    gen.manual_seed(21)
    codes = torch.randint(0, 16, (N, K), dtype=torch.int8, device="cuda", generator=gen)
    packed = dq.dq_hqq_pack(codes)
    del codes
    scl = dq.dq_hqq_group_major((torch.rand((N, K // 128), generator=gen, device="cuda") * 0.018 + 0.002).to(torch.bfloat16))
    zer = dq.dq_hqq_group_major((torch.rand((N, K // 128), generator=gen, device="cuda") * 3 + 6).to(torch.bfloat16))
    for M in (16, 1024):
        pause()
        x = randn((M, K), 1.0, 22 + M).to(torch.bfloat16)
        o = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        nws = dq.dq_hqq_workspace_size(M, N, K)
        ws = torch.zeros(nws, dtype=torch.uint8, device="cuda") if nws else None
        ms = _graph_ms(torch, lambda i, st: dq.dq_hqq_linear(x, packed, scl, zer, 128, out=o, workspace=ws, stream=st), n)
        nbytes = 2 * M * K + N * K // 2 + 2 * 2 * N * (K // 128) + 2 * M * N
        if M <= 128:
            e = _hbm_entry("dq_hqq_linear", ms, nbytes, peaks)
        else:
            tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
            e = dict(kernel="dq_hqq_linear", kernel_ms=round(ms, 5), bound="tensor", achieved=round(tf, 1),
                     unit="TFLOP/s", peak=peaks["bf16"], frac=round(tf / peaks["bf16"], 4), sm_mhz=_LAST_CLOCK[0])
        e["page_h100_ms"] = HQQ_PAGE_H100_MS[M]
        out[f"hqq_m{M}_4096x4096_g128"] = e
        del x, o, ws
    del packed, scl, zer
    torch.cuda.synchronize()
    assert dq.dq_sync_status() == dq.DQ_OK
    torch.cuda.empty_cache()
    # DRAM bytes per launch from the ncu capture of the bench workload of the
    # same kernel and shape (profiles/traffic.json; null when the kernel's
    # sources changed since)
    for tag, e in out.items():
        wl = next((w for pre, w in SECONDARY_TRAFFIC if tag.startswith(pre)), None)
        if wl is not None:
            e["traffic"] = measured_traffic(wl, e["kernel"])
            e["traffic_workload"] = wl
    return out


SECONDARY_TRAFFIC = (("quant_", "quant"), ("small_m16_", "small_m16"), ("large_m_", "large_m"),
                     ("vit_h_fc1_bsr10", "vit_fc1"), ("vit_h_fc2_bsr10", "vit_fc2"), ("s24_llm", "s24_llm"),
                     ("s24_small_m16", "s24_small_m16"), ("fp8_llm", "llm_fp8"), ("hqq_m16_", "hqq_m16"),
                     ("hqq_m1024_", "hqq_m1024"))


def run_e2e(args, wl, state, dq, torch, stream, ops, dom, world, max_over_ranks):
    """Same metric through the public API, host (pinned) buffers: every step
    copies its activations host->device and reads its result back
    device->host inside the timed region.  The three run as a pipeline on
    three streams: the copy-in of step i+1 (into the other of two device
    input buffers) overlaps step i's kernels, and step i's copy-out overlaps
    the copy-in of step i+2; a step's kernels wait for the previous step's
    copy-out (one device output buffer)."""
    copies = state["copies"]
    key = "x" if "x" in copies[0] else "A"
    bufs = [copies[0], copies[1 % len(copies)]]
    host_in = torch.empty(bufs[0][key].shape, dtype=bufs[0][key].dtype, pin_memory=True)
    host_in.copy_(bufs[0][key])
    outs = [state[n] for n, _ in state["d2h"]]
    host_outs = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
    K = args.steps
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
    in_done, comp_done = [ev(), ev()], [ev(), ev()]
    out_done = ev()
    state_first = {"done": False}

    def run(n_steps, start_ev=None):
        if start_ev is not None:
            s_in.wait_event(start_ev)
            s_out.wait_event(start_ev)
        for i in range(n_steps):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[b])          # step i-2 is done with this buffer
                bufs[b][key].copy_(host_in, non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if i >= 1 or state_first["done"]:
                stream.wait_event(out_done)                # the output buffer is free again
            state["step"](bufs[b], stream)
            comp_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[b])
                for o, h in zip(outs, host_outs):
                    h.copy_(o, non_blocking=True)
                out_done.record(s_out)
        state_first["done"] = True
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    run(3)
    torch.cuda.synchronize()
    st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st.record(stream)
    run(K, st)
    en.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(st.elapsed_time(en))
    h2d = sum(b for _, b in state["h2d"])
    d2h = sum(b for _, b in state["d2h"])
    if wl["kind"] == "quant":
        return dict(value=round(dom["bytes"] * world * K / (ms * 1e-3) / 1e9, 2), unit="GB/s",
                    h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h, pipelined=True)
    return dict(value=round(ops * world * K / (ms * 1e-3) / 1e12, 3),
                unit="TFLOP/s" if wl["kind"] == "hqq" else "TOPS",
                h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h, pipelined=True)


# ----------------------------------------------------------------------------
# CPU oracle: baseline / reference arm
# ----------------------------------------------------------------------------

def _oracle_sample(name, wl, d, rows):
    """Run the oracle on `rows` rows of the workload; return ops (or bytes)."""
    import numpy as np
    import oracle
    k = wl["kind"]
    if k in ("dense", "s24"):       # the 2:4 layer is the dense layer on the 2:4 weight
        if "_wq" not in d:
            d["_wq"], d["_sc"] = oracle.quantize_rows_f32(d["w"])
        x = d["x"][rows]
        q, s = oracle.quantize_rows_bf16(x)
        oracle.linear_bf16(q, s, d["_wq"], d["_sc"], d.get("bias"))
        return 2.0 * len(rows) * d["w"].shape[0] * d["w"].shape[1]
    if k == "gemm":
        acc = oracle.gemm_s32(d["a"][rows], d["b"])
        if wl.get("out") != "s32":
            oracle.epilogue_bf16(acc, d["s_row"][rows], d["s_col"])
        return 2.0 * len(rows) * d["b"].shape[0] * d["b"].shape[1]
    if k == "bsr":
        bs = wl.get("bs", 64)
        if "_vals" not in d:
            wq, sc = oracle.quantize_rows_f32(d["w"])
            d["_vals"], d["_sc"] = oracle.bsr_pack(wq, d["crow"], d["col"], bs), sc
        q, s = oracle.quantize_rows_bf16(d["x"][rows])
        acc = oracle.bsr_gemm_s32(q, d["N"], d["crow"], d["col"], d["_vals"], bs)
        oracle.epilogue_bf16(acc, s, d["_sc"])
        return 2.0 * len(rows) * int(d["crow"][-1]) * bs * bs
    if k == "quant":
        oracle.quantize_rows_bf16(d["x"][rows])
        return float(len(rows) * (3 * d["x"].shape[1] + 4))
    if k == "hqq":
        if "_w" not in d:
            d["_w"] = oracle.hqq_dequant(oracle.hqq_pack(d["codes"]), d["scale"], d["zero"], d["group"],
                                         signed=d["signed"])
        if wl.get("transposed"):
            oracle.hqq_linear_t_f64(d["x"][rows], d["_w"])
        else:
            oracle.hqq_linear_f64(d["x"][rows], d["_w"])
        return 2.0 * len(rows) * wl["N"] * wl["K"]
    raise ValueError(k)


def _rows_per_chunk(wl, d):
    k = wl["kind"]
    if k == "quant":
        return 256
    if k == "bsr":
        return 512
    return 8


def cpu_baseline(name, wl, d, budget_s=12.0):
    """The oracle, as it stands (single-threaded C), on a bounded sample of
    the workload: chunks of rows until ~budget_s of CPU work."""
    import numpy as np
    if "x" not in d and wl["kind"] in ("bsr",):
        import synth
        d = dict(d)
        d["x"] = synth.vit_h_bsr(0, wl["layer"], keep=wl.get("keep", 0.10), bs=wl.get("bs", 64))["x"]
    M = d["x"].shape[0] if "x" in d else d["a"].shape[0]
    chunk = _rows_per_chunk(wl, d)
    _oracle_sample(name, wl, d, np.arange(min(chunk, M)))    # prepare weights outside the clock
    done, units, t0 = 0, 0.0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s and done < M:
        rows = np.arange(done, min(M, done + chunk))
        units += _oracle_sample(name, wl, d, rows)
        done += len(rows)
    dt = time.perf_counter() - t0
    if wl["kind"] == "quant":
        v, unit = units / dt / 1e9, "GB/s"
    else:
        v, unit = units / dt / 1e12, "TFLOP/s" if wl["kind"] == "hqq" else "TOPS"
    return dict(value=round(v, 6), unit=unit, cores=1, kind="oracle",
                sample=f"first {done} of {M} rows of the same workload, {dt:.1f} s single-threaded "
                       f"(host: {os.cpu_count()} logical cores, oracle uses 1)")


def run_reference(args, rank, world):
    if rank != 0:
        return
    import numpy as np
    name = args.workload
    wl = WORKLOADS[name]
    d = _synth_inputs(name, wl, 0)
    M = d["x"].shape[0] if "x" in d else d["a"].shape[0]
    chunk = _rows_per_chunk(wl, d)
    _oracle_sample(name, wl, d, np.arange(min(chunk, M)))
    for i in range(args.warmup):
        _oracle_sample(name, wl, d, np.arange(min(chunk, M)))
    times, units = [], 0.0
    t_all = time.perf_counter()
    for i in range(args.steps):
        r0 = (i * chunk) % max(1, M - chunk + 1)
        rows = np.arange(r0, min(M, r0 + chunk))
        t0 = time.perf_counter()
        units += _oracle_sample(name, wl, d, rows)
        times.append(time.perf_counter() - t0)
    dt = time.perf_counter() - t_all
    if wl["kind"] == "quant":
        v, unit = units / dt / 1e9, "GB/s"
    else:
        v, unit = units / dt / 1e12, "TFLOP/s" if wl["kind"] == "hqq" else "TOPS"
    sample = f"{chunk} rows per step (of {M}), single-threaded C oracle on the host"
    line = dict(impl="reference", metric=METRIC, value=round(v, 6), unit=unit, n_gpus=world, steps=args.steps,
                warmup=args.warmup, ms_per_step=round(1e3 * dt / args.steps, 3), higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="int8", data="synthetic",
                config=dict(workload=wl["desc"]),
                cpu_baseline=dict(value=round(v, 6), unit=unit, cores=1, kind="oracle", sample=sample),
                e2e=dict(value=round(v, 6), unit=unit, h2d_bytes_per_step=0, d2h_bytes_per_step=0),
                gpu_launches=0)
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llm", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the issue-rate probe and the secondary workloads of the default run")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    main()

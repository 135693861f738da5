"""Python binding of libdq: the int8 dynamic-quantization linear layer on B200.

Argument marshalling only.  Every step of the layer runs in libdq's CUDA
kernels (``csrc/``); PyTorch supplies device memory and streams.  There is no
CPU or eager fallback: if ``libdq.so`` is missing, importing this package
raises, and every call on a non-sm_100 device returns an error.

Function names match the C ABI in ``include/dq.h``.  Tensors are torch CUDA
tensors; bf16 tensors are passed by pointer as 16-bit patterns.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdq.so")

DQ_OK, DQ_ERR_INVALID_ARG, DQ_ERR_UNSUPPORTED, DQ_ERR_CUDA, DQ_ERR_TIMEOUT = range(5)
DQ_OUT_BF16, DQ_OUT_S32, DQ_OUT_F32 = 0, 1, 2
DQ_HQQ_S4 = 1

# C prototypes: (name, restype, argtypes)
_P, _I64, _I32, _SZ, _U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
_PROTOS = {
    "dq_status_string": (ctypes.c_char_p, [_I32]),
    "dq_last_cuda_error": (_I32, []),
    "dq_version": (_I32, []),
    "dq_sync_status": (_I32, [_P]),
    "dq_set_wait_timeout_ns": (None, [_U64]),
    "dq_selftest_wait_timeout": (_I32, [_P]),
    "dq_quantize_rows": (_I32, [_P, _I64, _I64, _I64, _P, _I64, _P, _P]),
    "dq_quantize_weight": (_I32, [_P, _I64, _I64, _I64, _P, _I64, _P, _P]),
    "dq_int8_linear": (_I32, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _P, _I32, _P, _SZ, _P]),
    "dq_int8_linear_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "dq_int8_linear_noalloc": (_I32, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _P, _I32, _P]),
    "dq_bsr_int8_linear": (_I32, [_P, _P, _I64, _I64, _I64, _P, _P, _P, _I64, _P, _P, _P, _I32, _P]),
    "dq_bsr_pack": (_I32, [_P, _I64, _I64, _P, _P, _I64, _P, _P]),
    "dq_bsr_validate": (_I32, [_P, _P, _I64, _I64, _I64]),
    "dq_bsr_int8_linear_blocked": (_I32, [_P, _P, _I64, _I64, _I64, _I64, _P, _P, _P, _I64, _P, _P, _P, _I32,
                                          _P]),
    "dq_bsr_pack_blocked": (_I32, [_P, _I64, _I64, _I64, _P, _P, _I64, _P, _P]),
    "dq_bsr_validate_blocked": (_I32, [_P, _P, _I64, _I64, _I64, _I64]),
    "dq_mma_peak_probe": (_I32, [_I32, _I32, _P]),
    "dq_debug_set_schedule": (None, [_I32]),
    "dq_debug_set_tile_n": (None, [_I32]),
    "dq_quantize_rows_fp8": (_I32, [_P, _I64, _I64, _I64, _P, _I64, _P, _P]),
    "dq_quantize_weight_fp8": (_I32, [_P, _I64, _I64, _I64, _P, _I64, _P, _P]),
    "dq_fp8_linear": (_I32, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _P, _I32, _P]),
    "dq_debug_set_two_widths": (None, [_I32]),
    "dq_debug_set_bsr_panel": (None, [_I32]),
    "dq_debug_set_quant_kernel": (None, [_I32]),
    "dq_hqq_pack": (_I32, [_P, _I64, _I64, _P, _P]),
    "dq_hqq_dequantize": (_I32, [_P, _P, _P, _I64, _I64, _I32, _I32, _P, _P]),
    "dq_hqq_workspace_size": (_SZ, [_I64, _I64, _I64, _I32]),
    "dq_hqq_group_major": (_I32, [_P, _I64, _I64, _P, _P]),
    "dq_s24_compress": (_I32, [_P, _I64, _I64, _P, _P, _P, _P]),
    "dq_s24_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "dq_s24_int8_linear": (_I32, [_P, _P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _I32, _P, _SZ, _P]),
    "dq_hqq_linear": (_I32, [_P, _I64, _P, _P, _P, _I64, _I64, _I32, _I32, _P, _P, _SZ, _P]),
    "dq_hqq_linear_t": (_I32, [_P, _I64, _P, _P, _P, _I64, _I64, _I32, _I32, _P, _P, _SZ, _P]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libdq.so not found at {LIB_PATH}: build it with "
            "`python -m quantized_gemm_token_b200.build` (nvcc, sm_100a). "
            "There is no fallback implementation.")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _PROTOS.items():
        try:
            fn = getattr(lib, name)
        except AttributeError:
            raise ImportError(f"{LIB_PATH} is stale (no {name}): rebuild it with "
                              "`python -m quantized_gemm_token_b200.build`") from None
        fn.restype = res
        fn.argtypes = args
    return lib


class _MissingLibrary:
    """Stands in for libdq.so when it has not been built yet, so that the
    build module stays importable; every use raises."""

    def __init__(self, err: ImportError):
        self._err = err

    def __getattr__(self, name):
        raise ImportError(str(self._err))


try:
    lib = _load()
except ImportError as _e:
    lib = _MissingLibrary(_e)


class DQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.dq_status_string(status).decode()
        if status == DQ_ERR_CUDA:
            msg += f" (cudaError {lib.dq_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


def _check(status: int, where: str):
    if status != DQ_OK:
        raise DQError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _stream_obj(stream) -> torch.cuda.Stream:
    """The torch stream a layer call runs on (current stream when None; a raw
    cudaStream_t handle is wrapped)."""
    if stream is None:
        return torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream
    return torch.cuda.ExternalStream(int(stream))


def _scratch(shape, dtype, device, stream: torch.cuda.Stream, zero: bool = False) -> torch.Tensor:
    """Scratch a layer keeps between calls, allocated (and zero-filled) on the
    stream its kernels run on, so that the fill is ordered before them."""
    with torch.cuda.stream(stream):
        return (torch.zeros if zero else torch.empty)(shape, dtype=dtype, device=device)


def _used_on(stream: torch.cuda.Stream, *ts):
    """Tell the caching allocator that `stream` uses the cached scratch, so a
    later free or eviction waits for that stream's work."""
    for t in ts:
        if t is not None:
            t.record_stream(stream)


def _need(t: torch.Tensor, dtype, name: str, ndim: int = None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name}: expected a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got {t.dim()}")


def _contig(t: torch.Tensor, name: str):
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


# ---------------------------------------------------------------- status

def dq_status_string(status: int) -> str:
    return lib.dq_status_string(status).decode()


def dq_version() -> int:
    return lib.dq_version()


def dq_sync_status(stream=None) -> int:
    """Synchronise `stream` and return (and clear) the device error status."""
    return lib.dq_sync_status(_stream(stream))


def dq_set_wait_timeout_ns(ns: int) -> None:
    lib.dq_set_wait_timeout_ns(int(ns))


def dq_selftest_wait_timeout(stream=None) -> None:
    _check(lib.dq_selftest_wait_timeout(_stream(stream)), "dq_selftest_wait_timeout")


def dq_debug_set_schedule(mode: int) -> None:
    lib.dq_debug_set_schedule(int(mode))


def dq_debug_set_tile_n(n: int) -> None:
    lib.dq_debug_set_tile_n(int(n))


def dq_debug_set_two_widths(on: int) -> None:
    """Measurement knob: 0 turns off the two-width (wave-balanced) dense schedule."""
    lib.dq_debug_set_two_widths(int(on))


def dq_debug_set_bsr_panel(mode: int) -> None:
    """Measurement knob, BSR panel variant (K <= 1280): 0 never, 1 automatic, 2 always."""
    lib.dq_debug_set_bsr_panel(int(mode))


def dq_debug_set_quant_kernel(mode: int) -> None:
    lib.dq_debug_set_quant_kernel(int(mode))


# ---------------------------------------------------------------- quantize

def dq_quantize_rows(x: torch.Tensor, q: torch.Tensor = None, scales: torch.Tensor = None, stream=None):
    """Per-token int8 quantization: x bf16 [M, K] (row stride x.stride(0))
    -> (q int8 [M, K], scales fp32 [M])."""
    _need(x, torch.bfloat16, "x", 2)
    if x.stride(1) != 1:
        raise ValueError("x: rows must be contiguous")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty((M,), dtype=torch.float32, device=x.device)
    _need(q, torch.int8, "q", 2)
    _need(scales, torch.float32, "scales", 1)
    if q.stride(1) != 1 or tuple(q.shape) != (M, K) or scales.numel() != M:
        raise ValueError("q / scales: shape or layout mismatch")
    _check(lib.dq_quantize_rows(_ptr(x), M, K, x.stride(0), _ptr(q), q.stride(0), _ptr(scales),
                                _stream(stream)), "dq_quantize_rows")
    return q, scales


def dq_quantize_weight(w: torch.Tensor, wq: torch.Tensor = None, s_col: torch.Tensor = None, stream=None):
    """Per-output-channel int8 weight: w fp32 [N, K] -> (wq int8 [N, K], s_col fp32 [N])."""
    _need(w, torch.float32, "w", 2)
    if w.stride(1) != 1:
        raise ValueError("w: rows must be contiguous")
    N, K = w.shape
    if wq is None:
        wq = torch.empty((N, K), dtype=torch.int8, device=w.device)
    if s_col is None:
        s_col = torch.empty((N,), dtype=torch.float32, device=w.device)
    _check(lib.dq_quantize_weight(_ptr(w), N, K, w.stride(0), _ptr(wq), wq.stride(0), _ptr(s_col),
                                  _stream(stream)), "dq_quantize_weight")
    return wq, s_col


def dq_quantize_rows_fp8(x: torch.Tensor, q: torch.Tensor = None, scales: torch.Tensor = None, stream=None):
    """Per-token dynamic FP8: x bf16 [M, K] -> (q e4m3 codes uint8 [M, K], scales fp32 [M]),
    s = max(absmax, 1e-8) / 448, q = e4m3(clamp(x / s, -448, 448))."""
    _need(x, torch.bfloat16, "x", 2)
    if x.stride(1) != 1:
        raise ValueError("x: rows must be contiguous")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((M,), dtype=torch.float32, device=x.device)
    _need(q, torch.uint8, "q", 2)
    _need(scales, torch.float32, "scales", 1)
    if q.stride(1) != 1 or tuple(q.shape) != (M, K) or scales.numel() != M:
        raise ValueError("q / scales: shape or layout mismatch")
    _check(lib.dq_quantize_rows_fp8(_ptr(x), M, K, x.stride(0), _ptr(q), q.stride(0), _ptr(scales),
                                    _stream(stream)), "dq_quantize_rows_fp8")
    return q, scales


def dq_quantize_weight_fp8(w: torch.Tensor, wq: torch.Tensor = None, s_col: torch.Tensor = None, stream=None):
    """Per-output-channel FP8 weight: w fp32 [N, K] -> (wq e4m3 codes uint8 [N, K], s_col fp32 [N])."""
    _need(w, torch.float32, "w", 2)
    if w.stride(1) != 1:
        raise ValueError("w: rows must be contiguous")
    N, K = w.shape
    if wq is None:
        wq = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    if s_col is None:
        s_col = torch.empty((N,), dtype=torch.float32, device=w.device)
    _check(lib.dq_quantize_weight_fp8(_ptr(w), N, K, w.stride(0), _ptr(wq), wq.stride(0), _ptr(s_col),
                                      _stream(stream)), "dq_quantize_weight_fp8")
    return wq, s_col


def dq_fp8_linear(A, s_row, W, s_col, bias=None, out=None, out_dtype="bf16", stream=None):
    """FP8 sibling of dq_int8_linear: A, W e4m3 codes (uint8) [M, K], [N, K];
    out = bf16(acc * s_row * s_col + bias), or the fp32 accumulators with out_dtype="f32"."""
    if out_dtype in ("f32", "float32", torch.float32, DQ_OUT_F32):
        code = DQ_OUT_F32
    elif out_dtype in ("bf16", torch.bfloat16, DQ_OUT_BF16):
        code = DQ_OUT_BF16
    else:
        raise ValueError(f"out_dtype {out_dtype!r}")
    _need(A, torch.uint8, "A", 2)
    _need(W, torch.uint8, "W", 2)
    _contig(A, "A")
    _contig(W, "W")
    M, K = A.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("A and W disagree on K")
    if code == DQ_OUT_BF16:
        _need(s_row, torch.float32, "s_row", 1)
        _need(s_col, torch.float32, "s_col", 1)
        if s_row.numel() != M or s_col.numel() != N:
            raise ValueError("scale length mismatch")
    if bias is not None:
        _need(bias, torch.bfloat16, "bias", 1)
    odt = torch.bfloat16 if code == DQ_OUT_BF16 else torch.float32
    if out is None:
        out = torch.empty((M, N), dtype=odt, device=A.device)
    _need(out, odt, "out", 2)
    _contig(out, "out")
    _check(lib.dq_fp8_linear(_ptr(A), _ptr(s_row), M, K, _ptr(W), _ptr(s_col), N, _ptr(bias), _ptr(out),
                             code, _stream(stream)), "dq_fp8_linear")
    return out


# ---------------------------------------------------------------- linear

def _out_code(out_dtype) -> int:
    if out_dtype in ("bf16", torch.bfloat16, DQ_OUT_BF16):
        return DQ_OUT_BF16
    if out_dtype in ("s32", "int32", torch.int32, DQ_OUT_S32):
        return DQ_OUT_S32
    raise ValueError(f"out_dtype {out_dtype!r}")


def dq_int8_linear_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib.dq_int8_linear_workspace_size(M, N, K))


def _linear_args(A, s_row, W, s_col, bias, out, code, out_required: bool):
    """The checks of the dense int8 linear's arguments; returns (M, K, N, out)."""
    _need(A, torch.int8, "A", 2)
    _need(W, torch.int8, "W", 2)
    _contig(A, "A")
    _contig(W, "W")
    M, K = A.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("A and W disagree on K")
    if code == DQ_OUT_BF16:
        _need(s_row, torch.float32, "s_row", 1)
        _need(s_col, torch.float32, "s_col", 1)
        _contig(s_row, "s_row")
        _contig(s_col, "s_col")
        if s_row.numel() != M or s_col.numel() != N:
            raise ValueError("scale length mismatch")
    if bias is not None:
        _need(bias, torch.bfloat16, "bias", 1)
        _contig(bias, "bias")
        if bias.numel() != N:
            raise ValueError("bias length mismatch")
    odt = torch.bfloat16 if code == DQ_OUT_BF16 else torch.int32
    if out is None:
        if out_required:
            raise ValueError("out: a preallocated output tensor is required")
        out = torch.empty((M, N), dtype=odt, device=A.device)
    _need(out, odt, "out", 2)
    _contig(out, "out")
    if tuple(out.shape) != (M, N):
        raise ValueError(f"out: expected shape {(M, N)}, got {tuple(out.shape)}")
    return M, K, N, out


def dq_int8_linear(A, s_row, W, s_col, bias=None, out=None, out_dtype="bf16", workspace=None, stream=None):
    """out[M, N] = bf16(acc * s_row * s_col + bias), acc = A @ W^T exactly
    (or acc itself as int32 with out_dtype="s32").  `workspace` is an
    optional zero-filled uint8 CUDA tensor (see dq_int8_linear_workspace_size)."""
    code = _out_code(out_dtype)
    M, K, N, out = _linear_args(A, s_row, W, s_col, bias, out, code, out_required=False)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _need(workspace, torch.uint8, "workspace")
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel()
    _check(lib.dq_int8_linear(_ptr(A), _ptr(s_row), M, K, _ptr(W), _ptr(s_col), N, _ptr(bias), _ptr(out),
                              code, ws_ptr, ws_bytes, _stream(stream)), "dq_int8_linear")
    return out


DQ_NOALLOC_SCRATCH_BYTES = 32 << 20


def dq_int8_linear_noalloc(A, s_row, W, s_col, out, bias=None, out_dtype="bf16", stream=None):
    """dq_int8_linear for callers that cannot allocate device memory: the
    split-K scratch comes from libdq's static 32 MiB device array and the
    caller passes a preallocated `out` ([M, N], bf16 or int32 to match
    out_dtype); the arguments are checked as for dq_int8_linear.  Calls that
    overlap on the GPU race on that array; the first call on a device that
    uses it must come before any stream capture."""
    code = _out_code(out_dtype)
    M, K, N, out = _linear_args(A, s_row, W, s_col, bias, out, code, out_required=True)
    _check(lib.dq_int8_linear_noalloc(_ptr(A), _ptr(s_row), M, K, _ptr(W), _ptr(s_col), N, _ptr(bias),
                                      _ptr(out), code, _stream(stream)), "dq_int8_linear_noalloc")
    return out


def dq_bsr_int8_linear(A, s_row, N, crow, col, values, s_col, bias=None, out=None, out_dtype="bf16",
                       stream=None):
    """BSR variant of dq_int8_linear; W given as crow int32 [N/b+1], col int32
    [nnzb], values int8 [nnzb, b, b] with the block size b in {64, 32, 16}
    taken from values' shape (dq_bsr_int8_linear_blocked; b = 64 is
    dq_bsr_int8_linear)."""
    code = _out_code(out_dtype)
    _need(A, torch.int8, "A", 2)
    _contig(A, "A")
    M, K = A.shape
    _need(crow, torch.int32, "crow", 1)
    _need(col, torch.int32, "col", 1)
    _need(values, torch.int8, "values", 3)
    _contig(values, "values")
    nnzb, b = values.shape[0], values.shape[1]
    if values.shape[2] != b or N % b != 0 or crow.numel() != N // b + 1 or col.numel() != nnzb:
        raise ValueError("BSR arrays do not match N / nnzb / block size")
    if code == DQ_OUT_BF16:
        _need(s_row, torch.float32, "s_row", 1)
        _need(s_col, torch.float32, "s_col", 1)
    if bias is not None:
        _need(bias, torch.bfloat16, "bias", 1)
    odt = torch.bfloat16 if code == DQ_OUT_BF16 else torch.int32
    if out is None:
        out = torch.empty((M, N), dtype=odt, device=A.device)
    _need(out, odt, "out", 2)
    _contig(out, "out")
    vp = _ptr(values) if nnzb else None
    if b == 64:
        st = lib.dq_bsr_int8_linear(_ptr(A), _ptr(s_row), M, K, N, _ptr(crow), _ptr(col), vp, nnzb,
                                    _ptr(s_col), _ptr(bias), _ptr(out), code, _stream(stream))
        _check(st, "dq_bsr_int8_linear")
    else:
        st = lib.dq_bsr_int8_linear_blocked(_ptr(A), _ptr(s_row), M, K, N, b, _ptr(crow), _ptr(col), vp, nnzb,
                                            _ptr(s_col), _ptr(bias), _ptr(out), code, _stream(stream))
        _check(st, "dq_bsr_int8_linear_blocked")
    return out


def dq_bsr_pack(wq, crow, col, values=None, stream=None, block: int = 64):
    """Gather the block x block blocks of a dense int8 weight [N, K] named by (crow, col)."""
    _need(wq, torch.int8, "wq", 2)
    _contig(wq, "wq")
    N, K = wq.shape
    nnzb = col.numel()
    if values is None:
        values = torch.empty((nnzb, block, block), dtype=torch.int8, device=wq.device)
    _check(lib.dq_bsr_pack_blocked(_ptr(wq), N, K, block, _ptr(crow), _ptr(col), nnzb,
                                   _ptr(values) if nnzb else None, _stream(stream)), "dq_bsr_pack_blocked")
    return values


def dq_bsr_validate(crow, col, N: int, K: int, block: int = 64) -> int:
    return lib.dq_bsr_validate_blocked(_ptr(crow), _ptr(col) if col.numel() else None, N, K, block, col.numel())


def dq_mma_peak_probe(grid: int, iters: int, stream=None) -> None:
    _check(lib.dq_mma_peak_probe(grid, iters, _stream(stream)), "dq_mma_peak_probe")


# ---------------------------------------------------------------- int4 (HQQ)

def dq_hqq_pack(codes: torch.Tensor, packed: torch.Tensor = None, stream=None) -> torch.Tensor:
    """int4 codes int8 [R, C] (u4 0..15 or s4 -8..7) -> packed uint8 [R, C/2]
    (byte j = code 2j | code 2j+1 << 4)."""
    _need(codes, torch.int8, "codes", 2)
    _contig(codes, "codes")
    R, C = codes.shape
    if packed is None:
        packed = torch.empty((R, C // 2), dtype=torch.uint8, device=codes.device)
    _need(packed, torch.uint8, "packed", 2)
    _contig(packed, "packed")
    if tuple(packed.shape) != (R, C // 2):
        raise ValueError("packed must be [R, C/2]")
    _check(lib.dq_hqq_pack(_ptr(codes), R, C, _ptr(packed), _stream(stream)), "dq_hqq_pack")
    return packed


def dq_hqq_group_major(meta: torch.Tensor, out: torch.Tensor = None, stream=None) -> torch.Tensor:
    """Per-channel scales or zero points bf16 [N, K/group] -> the group-major
    [K/group, N] layout the int4 kernels read."""
    _need(meta, torch.bfloat16, "meta", 2)
    _contig(meta, "meta")
    N, G = meta.shape
    if out is None:
        out = torch.empty((G, N), dtype=torch.bfloat16, device=meta.device)
    _need(out, torch.bfloat16, "out", 2)
    _contig(out, "out")
    if tuple(out.shape) != (G, N):
        raise ValueError("out must be [G, N]")
    _check(lib.dq_hqq_group_major(_ptr(meta), N, G, _ptr(out), _stream(stream)), "dq_hqq_group_major")
    return out


def _hqq_weights(packed, scale, zero, group):
    _need(packed, torch.uint8, "packed", 2)
    _need(scale, torch.bfloat16, "scale", 2)
    _need(zero, torch.bfloat16, "zero", 2)
    for t, n in ((packed, "packed"), (scale, "scale"), (zero, "zero")):
        _contig(t, n)
    N, K = packed.shape[0], packed.shape[1] * 2
    if group <= 0 or K % group != 0:
        raise ValueError("group must divide K")
    if tuple(scale.shape) != (K // group, N) or tuple(zero.shape) != (K // group, N):
        raise ValueError("scale and zero must be group-major [K/group, N]")
    return N, K


def dq_hqq_dequantize(packed, scale, zero, group: int, signed: bool = False, out=None, stream=None):
    """w bf16 [N, K] = bf16(bf16(q - zero) * scale), per group of K (scale and
    zero group-major [K/group, N])."""
    N, K = _hqq_weights(packed, scale, zero, group)
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=packed.device)
    _need(out, torch.bfloat16, "out", 2)
    _contig(out, "out")
    _check(lib.dq_hqq_dequantize(_ptr(packed), _ptr(scale), _ptr(zero), N, K, group,
                                 DQ_HQQ_S4 if signed else 0, _ptr(out), _stream(stream)), "dq_hqq_dequantize")
    return out


def dq_hqq_workspace_size(M: int, N: int, K: int, transposed: bool = False) -> int:
    return int(lib.dq_hqq_workspace_size(M, N, K, int(transposed)))


def _hqq_call(fn, name, x, packed, scale, zero, group, signed, out, workspace, stream, transposed):
    N, K = _hqq_weights(packed, scale, zero, group)
    _need(x, torch.bfloat16, "x", 2)
    _contig(x, "x")
    M = x.shape[0]
    if x.shape[1] != (N if transposed else K):
        raise ValueError("activation width does not match the weight")
    n_out = K if transposed else N
    if out is None:
        out = torch.empty((M, n_out), dtype=torch.bfloat16, device=x.device)
    _need(out, torch.bfloat16, "out", 2)
    _contig(out, "out")
    if tuple(out.shape) != (M, n_out):
        raise ValueError("out shape")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _need(workspace, torch.uint8, "workspace")
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel()
    _check(fn(_ptr(x), M, _ptr(packed), _ptr(scale), _ptr(zero), N, K, group, DQ_HQQ_S4 if signed else 0,
              _ptr(out), ws_ptr, ws_bytes, _stream(stream)), name)
    return out


def dq_hqq_linear(x, packed, scale, zero, group: int, signed: bool = False, out=None, workspace=None,
                  stream=None):
    """out[M, N] = x[M, K] @ w^T with w the dequantized int4 weight [N, K]
    (dequantization fused into the tensor-core GEMM).  `workspace` is
    accepted and unused: few-token calls split the contraction over a
    cluster of CTAs that reduce through distributed shared memory
    (dq_hqq_workspace_size returns 0)."""
    return _hqq_call(lib.dq_hqq_linear, "dq_hqq_linear", x, packed, scale, zero, group, signed, out,
                     workspace, stream, False)


def dq_hqq_linear_t(y, packed, scale, zero, group: int, signed: bool = False, out=None, workspace=None,
                    stream=None):
    """out[M, K] = y[M, N] @ w (the transposed product, for the input gradient)."""
    return _hqq_call(lib.dq_hqq_linear_t, "dq_hqq_linear_t", y, packed, scale, zero, group, signed, out,
                     workspace, stream, True)


class HqqLinear:
    """Weight-only int4 linear: packed u4 / s4 codes with bf16 scale and zero
    point per group of in-features (held group-major, [K/group, N]).
    forward(x) = x @ w^T, backward_input(g) = g @ w.  No workspace: the
    few-token split contraction reduces inside a cluster of CTAs."""

    def __init__(self, packed, scale, zero, group: int, signed: bool = False):
        self.packed, self.scale, self.zero, self.group, self.signed = packed, scale, zero, group, signed
        self.N, self.K = packed.shape[0], packed.shape[1] * 2

    @classmethod
    def from_codes(cls, codes: torch.Tensor, scale, zero, group: int, signed: bool = False):
        """codes int8 [N, K]; scale, zero bf16 per channel [N, K/group]."""
        return cls(dq_hqq_pack(codes), dq_hqq_group_major(scale), dq_hqq_group_major(zero), group, signed)

    def __call__(self, x: torch.Tensor, out: torch.Tensor = None, stream=None):
        return dq_hqq_linear(x, self.packed, self.scale, self.zero, self.group, self.signed, out=out,
                             stream=stream)

    def backward_input(self, grad_out: torch.Tensor, out: torch.Tensor = None, stream=None):
        return dq_hqq_linear_t(grad_out, self.packed, self.scale, self.zero, self.group, self.signed, out=out,
                               stream=stream)


# ---------------------------------------------------------------- 2:4 sparse

def dq_s24_compress(wq: torch.Tensor, values: torch.Tensor = None, meta: torch.Tensor = None,
                    violations: torch.Tensor = None, stream=None):
    """2:4-sparse int8 weight [N, K] -> (values int8 [N, K/2], meta uint8 [N, K/8]).
    `violations` (int32 CUDA tensor of one element, optional) counts groups
    with more than two nonzeros."""
    _need(wq, torch.int8, "wq", 2)
    _contig(wq, "wq")
    N, K = wq.shape
    if values is None:
        values = torch.empty((N, K // 2), dtype=torch.int8, device=wq.device)
    if meta is None:
        meta = torch.empty((N, K // 8), dtype=torch.uint8, device=wq.device)
    _need(values, torch.int8, "values", 2)
    _need(meta, torch.uint8, "meta", 2)
    if violations is not None:
        _need(violations, torch.int32, "violations")
    _check(lib.dq_s24_compress(_ptr(wq), N, K, _ptr(values), _ptr(meta), _ptr(violations), _stream(stream)),
           "dq_s24_compress")
    return values, meta


def dq_s24_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib.dq_s24_workspace_size(M, N, K))


def dq_s24_int8_linear(A, s_row, values, meta, s_col, bias=None, out=None, out_dtype="bf16", workspace=None,
                       stream=None):
    """The int8 layer with a compressed 2:4 weight: out[M, N] = bf16(acc * s_row
    * s_col + bias), acc = A @ W^T exactly (W decompressed), or acc as int32.
    `workspace`: as for dq_hqq_linear (dq_s24_workspace_size, one per shape)."""
    code = _out_code(out_dtype)
    _need(A, torch.int8, "A", 2)
    _need(values, torch.int8, "values", 2)
    _need(meta, torch.uint8, "meta", 2)
    for t, n in ((A, "A"), (values, "values"), (meta, "meta")):
        _contig(t, n)
    M, K = A.shape
    N = values.shape[0]
    if values.shape[1] * 2 != K or tuple(meta.shape) != (N, K // 8):
        raise ValueError("values must be [N, K/2] and meta [N, K/8]")
    if code == DQ_OUT_BF16:
        _need(s_row, torch.float32, "s_row", 1)
        _need(s_col, torch.float32, "s_col", 1)
    if bias is not None:
        _need(bias, torch.bfloat16, "bias", 1)
    odt = torch.bfloat16 if code == DQ_OUT_BF16 else torch.int32
    if out is None:
        out = torch.empty((M, N), dtype=odt, device=A.device)
    _need(out, odt, "out", 2)
    _contig(out, "out")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _need(workspace, torch.uint8, "workspace")
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel()
    _check(lib.dq_s24_int8_linear(_ptr(A), _ptr(s_row), M, K, _ptr(values), _ptr(meta), _ptr(s_col), N, _ptr(bias),
                                  _ptr(out), code, ws_ptr, ws_bytes, _stream(stream)), "dq_s24_int8_linear")
    return out


# ---------------------------------------------------------------- layer

class Int8DynamicLinear:
    """The layer: per-token dynamic int8 quantization of bf16 activations,
    then the fused i8i8->bf16 GEMM against a per-channel int8 weight (dense,
    or 64x64 BSR when built with from_bsr).  Holds the quantized weight, the
    activation scratch and the stream-K workspace; call it on bf16 [M, K]."""

    def __init__(self, wq, s_col, bias=None, bsr=None):
        self.wq, self.s_col, self.bias, self.bsr = wq, s_col, bias, bsr
        self.N = s_col.numel()
        self.K = wq.shape[1] if bsr is None else bsr["K"]
        self._q = self._s = self._ws = None

    @classmethod
    def from_float(cls, w: torch.Tensor, bias: torch.Tensor = None):
        wq, s_col = dq_quantize_weight(w)
        return cls(wq, s_col, bias)

    @classmethod
    def from_bsr(cls, w_masked: torch.Tensor, crow: torch.Tensor, col: torch.Tensor, bias=None):
        """w_masked: fp32 [N, K] already zero outside the kept 64x64 blocks."""
        wq, s_col = dq_quantize_weight(w_masked)
        values = dq_bsr_pack(wq, crow, col)
        return cls(None, s_col, bias, dict(crow=crow, col=col, values=values, K=w_masked.shape[1]))

    def _buffers(self, M, device, st):
        if self._q is None or self._q.shape[0] < M:
            self._q = _scratch((M, self.K), torch.int8, device, st)
            self._s = _scratch((M,), torch.float32, device, st)
        if self.bsr is None:
            n = dq_int8_linear_workspace_size(M, self.N, self.K)
            if n and (self._ws is None or self._ws.numel() < n):
                self._ws = _scratch((n,), torch.uint8, device, st, zero=True)
        return self._q[:M], self._s[:M]

    def __call__(self, x: torch.Tensor, out: torch.Tensor = None, stream=None):
        M = x.shape[0]
        st = _stream_obj(stream)
        q, s = self._buffers(M, x.device, st)
        dq_quantize_rows(x, q, s, stream=st)
        if self.bsr is None:
            ws = self._ws
            if ws is not None and ws.numel() < dq_int8_linear_workspace_size(M, self.N, self.K):
                ws = None
            y = dq_int8_linear(q, s, self.wq, self.s_col, self.bias, out=out, workspace=ws, stream=st)
        else:
            b = self.bsr
            y = dq_bsr_int8_linear(q, s, self.N, b["crow"], b["col"], b["values"], self.s_col, self.bias,
                                   out=out, stream=st)
        _used_on(st, self._q, self._s, self._ws)
        return y


class S24Int8Linear:
    """The int8 dynamic-quantization layer with a 2:4-sparse weight: the fp32
    weight (already 2:4 sparse) is quantized per channel and compressed once;
    each call quantizes the bf16 activations per token and runs the
    compressed-weight GEMM with the fused epilogue.  Split workspaces are kept
    per token count (a workspace serves one shape)."""

    def __init__(self, values, meta, s_col, bias=None):
        self.values, self.meta, self.s_col, self.bias = values, meta, s_col, bias
        self.N, self.K = values.shape[0], values.shape[1] * 2
        self._q = self._s = None
        self._ws = {}

    @classmethod
    def from_float(cls, w: torch.Tensor, bias: torch.Tensor = None, violations: torch.Tensor = None):
        """w: fp32 [N, K] with at most two nonzeros in every four consecutive
        in-features (`violations`, optional int32 CUDA tensor, counts the
        groups that have more)."""
        wq, s_col = dq_quantize_weight(w)
        values, meta = dq_s24_compress(wq, violations=violations)
        return cls(values, meta, s_col, bias)

    def __call__(self, x: torch.Tensor, out: torch.Tensor = None, stream=None):
        M = x.shape[0]
        st = _stream_obj(stream)
        if self._q is None or self._q.shape[0] < M:
            self._q = _scratch((M, self.K), torch.int8, x.device, st)
            self._s = _scratch((M,), torch.float32, x.device, st)
        q, s = self._q[:M], self._s[:M]
        dq_quantize_rows(x, q, s, stream=st)
        if M not in self._ws:
            if len(self._ws) >= 16:                 # keep the most recent shapes only
                self._ws.pop(next(iter(self._ws)))
            n = dq_s24_workspace_size(M, self.N, self.K)
            self._ws[M] = _scratch((n,), torch.uint8, x.device, st, zero=True) if n else None
        y = dq_s24_int8_linear(q, s, self.values, self.meta, self.s_col, self.bias, out=out,
                               workspace=self._ws[M], stream=st)
        _used_on(st, self._q, self._s, self._ws[M])
        return y

"""CPU oracle for the int8 dynamic-quantization linear layer (numpy front end).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product path (``quantized_gemm_token_b200``) never does, and this package
never imports the product.

The arithmetic lives in ``dq_oracle.c`` (plain single-threaded C); this
module only marshals numpy arrays.  bf16 tensors are carried as their uint16
bit patterns.

What each routine follows (page titles and parts; the FP8 routines follow the
vLLM csrc/quantization commits: dynamic scales, clamp to the e4m3 range):
  * quantize_rows_bf16 / quantize_rows_f32 -- per-token (per-row) absmax int8
    dynamic quantization: "int8 dynamic quant + bsr support" (pytorch/ao PR
    821, description); absmax/127 symmetric scale: "sparse_fc supported"
    (PaddlePaddle PR 41770, SpmmPluginDynamic constructor).  Scale
    s = max(absmax, 1e-8f)/127 in fp32, q = clamp(rint(x/s), -127, 127), ties
    to even.
  * gemm_s32 / gemm_s64 -- int8 x int8 -> int32 (PR 821 review: the dot
    accumulator is int32; overflow bound 2^31/2^14).
  * epilogue_bf16 -- out = bf16(acc * s_row * s_col + bias) (PR 821: i8i8->bf16
    keeps accuracy).
  * bsr_gemm_s32 / bsr_pack / bsr_densify -- 64x64 BSR weight given as
    crow_indices / col_indices / values (PR 821 description; --bsr 64).
  * hqq_pack / hqq_unpack / hqq_dequant / hqq_linear_f64 / hqq_linear_t_f64 --
    weight-only int4 (u4 / s4) asymmetric groupwise dequantization fused into
    a bf16 matmul, forward and transposed ("Fused HQQ Quantization Gemm",
    pytorch/ao PR 153, description and implementation details):
    w = bf16(bf16(q - z) * s) per group of K.
  * s24_compress / s24_decompress -- 2:4 semi-structured sparse int8 weight
    ("sparse_fc supported", PaddlePaddle PR 41770: 2:4-sparse FC weights
    compressed on the device); the product is gemm_s32 on the decompressed
    weight, then epilogue_bf16.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int64
        lib.oracle_quantize_rows_bf16.argtypes = [P, I, I, I, P, I, P]
        lib.oracle_quantize_rows_bf16.restype = ctypes.c_int
        lib.oracle_quantize_rows_f32.argtypes = [P, I, I, I, P, I, P]
        lib.oracle_quantize_rows_f32.restype = ctypes.c_int
        lib.oracle_gemm_s32.argtypes = [P, I, I, I, P, I, I, P]
        lib.oracle_gemm_s64.argtypes = [P, I, I, I, P, I, I, P]
        lib.oracle_epilogue_bf16.argtypes = [P, I, I, P, P, P, P]
        lib.oracle_bsr_gemm_s32.argtypes = [P, I, I, I, I, P, P, P, I, P]
        lib.oracle_bsr_pack.argtypes = [P, I, I, P, P, I, P]
        lib.oracle_bsr_densify.argtypes = [I, I, P, P, P, I, P]
        lib.oracle_float_to_bf16.argtypes = [ctypes.c_float]
        lib.oracle_float_to_bf16.restype = ctypes.c_uint16
        lib.oracle_bf16_to_float.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_float.restype = ctypes.c_float
        lib.oracle_quantize_rows_bf16_fp8.argtypes = [P, I, I, I, P, I, P]
        lib.oracle_quantize_rows_bf16_fp8.restype = ctypes.c_int
        lib.oracle_quantize_rows_f32_fp8.argtypes = [P, I, I, I, P, I, P]
        lib.oracle_quantize_rows_f32_fp8.restype = ctypes.c_int
        lib.oracle_gemm_fp8_f64.argtypes = [P, I, I, I, P, I, I, P]
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = ctypes.c_double
        lib.oracle_float_to_e4m3.argtypes = [ctypes.c_float]
        lib.oracle_float_to_e4m3.restype = ctypes.c_uint8
        Ci = ctypes.c_int
        lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_double_to_bf16.restype = ctypes.c_uint16
        lib.oracle_hqq_pack.argtypes = [P, I, I, P]
        lib.oracle_hqq_unpack.argtypes = [P, I, I, Ci, P]
        lib.oracle_hqq_dequant.argtypes = [P, P, P, I, I, I, Ci, P]
        lib.oracle_hqq_linear_f64.argtypes = [P, P, I, I, I, P]
        lib.oracle_hqq_linear_t_f64.argtypes = [P, P, I, I, I, P]
        lib.oracle_s24_compress.argtypes = [P, I, I, P, P]
        lib.oracle_s24_compress.restype = ctypes.c_int64
        lib.oracle_s24_decompress.argtypes = [P, P, I, I, P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def quantize_rows_bf16(x_bits: np.ndarray):
    """x_bits: uint16 [M, K] (bf16 patterns) -> (q int8 [M, K], scales fp32 [M])."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    s = np.empty((M,), np.float32)
    rc = _load().oracle_quantize_rows_bf16(_ptr(x), M, K, K, _ptr(q), K, _ptr(s))
    if rc != 0:
        raise ValueError("row too long for the oracle")
    return q, s


def quantize_rows_f32(w: np.ndarray):
    """w: fp32 [N, K] -> (q int8 [N, K], per-row scales fp32 [N])."""
    w = _c(w, np.float32)
    N, K = w.shape
    q = np.empty((N, K), np.int8)
    s = np.empty((N,), np.float32)
    _load().oracle_quantize_rows_f32(_ptr(w), N, K, K, _ptr(q), K, _ptr(s))
    return q, s


def gemm_s32(A: np.ndarray, W: np.ndarray) -> np.ndarray:
    """A int8 [M, K], W int8 [N, K] -> int32 [M, N] = A @ W^T (exact)."""
    A = _c(A, np.int8)
    W = _c(W, np.int8)
    M, K = A.shape
    N = W.shape[0]
    assert W.shape[1] == K
    out = np.empty((M, N), np.int32)
    _load().oracle_gemm_s32(_ptr(A), M, K, K, _ptr(W), N, K, _ptr(out))
    return out


def gemm_s64(A: np.ndarray, W: np.ndarray) -> np.ndarray:
    A = _c(A, np.int8)
    W = _c(W, np.int8)
    M, K = A.shape
    N = W.shape[0]
    out = np.empty((M, N), np.int64)
    _load().oracle_gemm_s64(_ptr(A), M, K, K, _ptr(W), N, K, _ptr(out))
    return out


def epilogue_bf16(acc, s_row, s_col, bias_bits=None) -> np.ndarray:
    """acc int32 [M, N] -> bf16 bits uint16 [M, N]."""
    acc = _c(acc, np.int32)
    M, N = acc.shape
    s_row = _c(s_row, np.float32)
    s_col = _c(s_col, np.float32)
    out = np.empty((M, N), np.uint16)
    if bias_bits is not None:
        bias_bits = _c(bias_bits, np.uint16)
        bp = _ptr(bias_bits)
    else:
        bp = None
    _load().oracle_epilogue_bf16(_ptr(acc), M, N, _ptr(s_row), _ptr(s_col), bp, _ptr(out))
    return out


def bsr_gemm_s32(A, N, crow, col, values, bs=64) -> np.ndarray:
    A = _c(A, np.int8)
    M, K = A.shape
    crow = _c(crow, np.int32)
    col = _c(col, np.int32)
    values = _c(values, np.int8)
    out = np.empty((M, N), np.int32)
    _load().oracle_bsr_gemm_s32(_ptr(A), M, K, K, N, _ptr(crow), _ptr(col), _ptr(values),
                                bs, _ptr(out))
    return out


def bsr_pack(W, crow, col, bs=64) -> np.ndarray:
    W = _c(W, np.int8)
    N, K = W.shape
    crow = _c(crow, np.int32)
    col = _c(col, np.int32)
    nnzb = int(crow[-1])
    values = np.empty((nnzb, bs, bs), np.int8)
    _load().oracle_bsr_pack(_ptr(W), N, K, _ptr(crow), _ptr(col), bs, _ptr(values))
    return values


def bsr_densify(N, K, crow, col, values, bs=64) -> np.ndarray:
    crow = _c(crow, np.int32)
    col = _c(col, np.int32)
    values = _c(values, np.int8)
    out = np.empty((N, K), np.int32)
    _load().oracle_bsr_densify(N, K, _ptr(crow), _ptr(col), _ptr(values), bs, _ptr(out))
    return out


def linear_bf16(q, s_row, Wq, s_col, bias_bits=None):
    """Composition: exact GEMM then the fp32/bf16 epilogue."""
    return epilogue_bf16(gemm_s32(q, Wq), s_row, s_col, bias_bits)


def dynamic_linear_bf16(x_bits, Wq, s_col, bias_bits=None):
    """The full layer: per-token quantize, int8 GEMM, fused-epilogue math."""
    q, s_row = quantize_rows_bf16(x_bits)
    return linear_bf16(q, s_row, Wq, s_col, bias_bits), q, s_row


def float_to_bf16(f: float) -> int:
    return int(_load().oracle_float_to_bf16(float(f)))


def bf16_to_float(h: int) -> float:
    return float(_load().oracle_bf16_to_float(int(h)))


# ---------------------------------------------------------------- FP8 (e4m3)

def e4m3_to_float64(codes) -> np.ndarray:
    """e4m3 codes (uint8, any shape) -> their values (float64; NaN codes -> NaN)."""
    lib = _load()
    table = np.array([lib.oracle_e4m3_to_double(c) for c in range(256)], np.float64)
    return table[np.asarray(codes, np.uint8)]


def float_to_e4m3(x) -> np.ndarray:
    """finite fp32 values -> e4m3 codes (round to nearest even, magnitudes >= 448 -> 448)."""
    lib = _load()
    x = np.asarray(x, np.float32)
    return np.array([lib.oracle_float_to_e4m3(float(v)) for v in x.ravel()], np.uint8).reshape(x.shape)


def quantize_rows_bf16_fp8(x_bits: np.ndarray):
    """x_bits: uint16 [M, K] (bf16) -> (q e4m3 codes uint8 [M, K], scales fp32 [M]);
    s = fp32(max(absmax, 1e-8) / 448), q = e4m3(clamp(fp32(x / s), -448, 448))."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    s = np.empty((M,), np.float32)
    if _load().oracle_quantize_rows_bf16_fp8(_ptr(x), M, K, K, _ptr(q), K, _ptr(s)) != 0:
        raise MemoryError("oracle row buffer")
    return q, s


def quantize_rows_f32_fp8(w: np.ndarray):
    """w: fp32 [N, K] -> (q e4m3 codes uint8 [N, K], per-row scales fp32 [N])."""
    w = _c(w, np.float32)
    N, K = w.shape
    q = np.empty((N, K), np.uint8)
    s = np.empty((N,), np.float32)
    _load().oracle_quantize_rows_f32_fp8(_ptr(w), N, K, K, _ptr(q), K, _ptr(s))
    return q, s


def gemm_fp8_f64(A: np.ndarray, W: np.ndarray) -> np.ndarray:
    """A e4m3 [M, K], W e4m3 [N, K] (uint8 codes) -> float64 [M, N] = the exact A @ W^T."""
    A = _c(A, np.uint8)
    W = _c(W, np.uint8)
    M, K = A.shape
    N = W.shape[0]
    assert W.shape[1] == K
    out = np.empty((M, N), np.float64)
    _load().oracle_gemm_fp8_f64(_ptr(A), M, K, K, _ptr(W), N, K, _ptr(out))
    return out


def double_to_bf16(v: float) -> int:
    """float64 -> bf16 bit pattern, one rounding to nearest even."""
    return int(_load().oracle_double_to_bf16(float(v)))


def hqq_pack(codes: np.ndarray) -> np.ndarray:
    """int4 codes int8 [R, C] (u4 0..15 or s4 -8..7, C even) -> packed uint8 [R, C/2]:
    byte j = code[2j] | code[2j+1] << 4 (nibbles, two's complement for s4)."""
    c = _c(codes, np.int8)
    R, C = c.shape
    assert C % 2 == 0
    out = np.empty((R, C // 2), np.uint8)
    _load().oracle_hqq_pack(_ptr(c), R, C, _ptr(out))
    return out


def hqq_unpack(packed: np.ndarray, signed: bool = False) -> np.ndarray:
    """packed uint8 [R, C/2] -> codes int8 [R, C]."""
    p = _c(packed, np.uint8)
    R, H = p.shape
    out = np.empty((R, 2 * H), np.int8)
    _load().oracle_hqq_unpack(_ptr(p), R, 2 * H, int(signed), _ptr(out))
    return out


def hqq_dequant(packed, scale_bits, zero_bits, group: int, signed: bool = False) -> np.ndarray:
    """packed uint8 [N, K/2], scale / zero bf16 bits [N, K/group] -> w bf16 bits [N, K],
    w = bf16(bf16(q - z) * s)."""
    p = _c(packed, np.uint8)
    N, H = p.shape
    K = 2 * H
    assert K % group == 0
    sc = _c(scale_bits, np.uint16)
    ze = _c(zero_bits, np.uint16)
    assert sc.shape == (N, K // group) and ze.shape == (N, K // group)
    w = np.empty((N, K), np.uint16)
    _load().oracle_hqq_dequant(_ptr(p), _ptr(sc), _ptr(ze), N, K, group, int(signed), _ptr(w))
    return w


def hqq_linear_f64(x_bits, w_bits) -> np.ndarray:
    """x bf16 [M, K], w bf16 [N, K] -> float64 [M, N] = x @ w^T (exact products, double sums)."""
    x = _c(x_bits, np.uint16)
    w = _c(w_bits, np.uint16)
    M, K = x.shape
    N = w.shape[0]
    assert w.shape[1] == K
    out = np.empty((M, N), np.float64)
    _load().oracle_hqq_linear_f64(_ptr(x), _ptr(w), M, N, K, _ptr(out))
    return out


def hqq_linear_t_f64(y_bits, w_bits) -> np.ndarray:
    """y bf16 [M, N], w bf16 [N, K] -> float64 [M, K] = y @ w (the transposed product)."""
    y = _c(y_bits, np.uint16)
    w = _c(w_bits, np.uint16)
    M, N = y.shape
    K = w.shape[1]
    assert w.shape[0] == N
    out = np.empty((M, K), np.float64)
    _load().oracle_hqq_linear_t_f64(_ptr(y), _ptr(w), M, N, K, _ptr(out))
    return out


def s24_compress(W: np.ndarray):
    """Wq int8 [N, K] (K % 8 == 0) -> (values int8 [N, K/2], meta uint8 [N, K/8], groups with > 2 nonzeros)."""
    W = _c(W, np.int8)
    N, K = W.shape
    assert K % 8 == 0
    values = np.empty((N, K // 2), np.int8)
    meta = np.zeros((N, K // 8), np.uint8)
    bad = _load().oracle_s24_compress(_ptr(W), N, K, _ptr(values), _ptr(meta))
    return values, meta, int(bad)


def s24_decompress(values: np.ndarray, meta: np.ndarray) -> np.ndarray:
    """(values [N, K/2], meta [N, K/8]) -> Wq int8 [N, K]."""
    v = _c(values, np.int8)
    m = _c(meta, np.uint8)
    N, H = v.shape
    K = 2 * H
    assert m.shape == (N, K // 8)
    W = np.empty((N, K), np.int8)
    _load().oracle_s24_decompress(_ptr(v), _ptr(m), N, K, _ptr(W))
    return W

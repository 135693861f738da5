"""Seeded synthetic inputs for the int8 dynamic-quantization linear layer.

This module only draws random numbers and builds index structures.  It holds
none of the method's arithmetic (no absmax, no scale, no rounding to int8, no
GEMM): both the CPU oracle's tests and the CUDA path's tests and benchmark use
it, and it imports neither of them.

Recipe (one per tensor, all in fp32 before any bf16 rounding):
  * generator: numpy ``Generator(Philox(key=seed))``; sub-seeds per tensor:
    X = seed, W = seed+1, bias = seed+2, block mask = seed+3, outlier
    channels = seed+4, scales = seed+5 / seed+6.
  * "N(0, sigma)" means mean 0 and standard deviation sigma (the nn.Linear
    init convention): an fp32 standard normal times fp32(sigma).
  * bf16 tensors: the fp32 draw rounded once to bf16 (round to nearest, ties
    to even) and carried as uint16 bit patterns.
  * outlier channels: round(frac * K) distinct channels from a seeded
    permutation, the same for every row, multiplied by 20 in fp32 before the
    bf16 rounding.
  * BSR mask: exactly round(keep * nblocks) blocks drawn uniformly without
    replacement, column indices sorted inside each block row.
"""
from __future__ import annotations

import numpy as np


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=int(seed)))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); return uint16 patterns.
    Inputs are finite draws, so no NaN/inf handling is needed here."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_f32(shape, sigma: float, seed: int) -> np.ndarray:
    z = rng(seed).standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        z *= np.float32(sigma)
    return z


def normal_bf16(shape, sigma: float, seed: int) -> np.ndarray:
    return f32_to_bf16_bits(normal_f32(shape, sigma, seed))


def uniform_int8(shape, lo: int, hi: int, seed: int) -> np.ndarray:
    return rng(seed).integers(lo, hi + 1, size=shape, dtype=np.int16).astype(np.int8)


def uniform_f32(shape, lo: float, hi: float, seed: int) -> np.ndarray:
    return rng(seed).uniform(lo, hi, size=shape).astype(np.float32)


def outlier_channels(K: int, frac: float, seed: int) -> np.ndarray:
    n = int(round(frac * K))
    return np.sort(rng(seed).permutation(K)[:n]).astype(np.int64)


def bsr_pattern(n_block_rows: int, n_block_cols: int, keep: float, seed: int):
    """Uniform random block mask keeping exactly round(keep * nblocks)
    blocks.  Returns (crow int32 [nbr+1], col int32 [nnzb])."""
    total = n_block_rows * n_block_cols
    nnzb = int(round(keep * total))
    chosen = np.sort(rng(seed).choice(total, size=nnzb, replace=False))
    rows = chosen // n_block_cols
    cols = chosen % n_block_cols
    counts = np.bincount(rows, minlength=n_block_rows)
    crow = np.zeros(n_block_rows + 1, np.int32)
    crow[1:] = np.cumsum(counts)
    return crow, cols.astype(np.int32)


def block_mask_dense(N: int, K: int, crow, col, bs: int = 64) -> np.ndarray:
    """bool [N, K]: True inside the kept blocks."""
    m = np.zeros((N // bs, K // bs), bool)
    for b in range(N // bs):
        m[b, col[crow[b]:crow[b + 1]]] = True
    return np.repeat(np.repeat(m, bs, axis=0), bs, axis=1)


# --------------------------------------------------------------------------
# The workloads.  Each returns plain numpy arrays; the caller quantizes the
# weight (oracle or library) and moves data where it needs it.
# --------------------------------------------------------------------------

def tiny(seed: int = 0):
    """X bf16 [64, 256] ~ N(0,1); W fp32 [256, 256] ~ N(0,0.02); bias bf16
    [256] ~ N(0,0.1); out bf16 [64, 256]."""
    return dict(name="tiny dense M=64 K=256 N=256",
                x=normal_bf16((64, 256), 1.0, seed),
                w=normal_f32((256, 256), 0.02, seed + 1),
                bias=normal_bf16((256,), 0.1, seed + 2))


def llm(seed: int = 0, M: int = 2048, K: int = 4096, N: int = 4096):
    """X bf16 [M, K] ~ N(0,1) with 1% of the K channels x20 (same channels in
    every row); W fp32 [N, K] ~ N(0,0.02); no bias."""
    x = normal_f32((M, K), 1.0, seed)
    ch = outlier_channels(K, 0.01, seed + 4)
    x[:, ch] *= np.float32(20.0)
    return dict(name=f"LLM dense M={M} K={K} N={N} (1% x20 outlier channels)",
                x=f32_to_bf16_bits(x), w=normal_f32((N, K), 0.02, seed + 1),
                bias=None, outliers=ch)


def large_m(seed: int = 0, M: int = 38400, K: int = 1024, N: int = 4096):
    """A int8 [M, K], B int8 [N, K] uniform in [-127, 127]; fp32 row/col
    scales U(0.001, 0.05)."""
    return dict(name=f"large-M int8 GEMM M={M} K={K} N={N}",
                a=uniform_int8((M, K), -127, 127, seed),
                b=uniform_int8((N, K), -127, 127, seed + 1),
                s_row=uniform_f32((M,), 0.001, 0.05, seed + 5),
                s_col=uniform_f32((N,), 0.001, 0.05, seed + 6))


def vit_h_bsr(seed: int = 0, layer: str = "fc1", M: int = 256 * 257, keep: float = 0.10,
              bs: int = 64, with_x: bool = True):
    """ViT-H/14 MLP at batch 256 (257 tokens per image): fc1 K=1280 -> N=5120,
    fc2 K=5120 -> N=1280.  X bf16 ~ N(0,1); W ~ N(0,0.02) masked to a uniform
    random fraction `keep` (10 % by default; the PR 821 benchmark keeps 20 %)
    of its bs x bs blocks (masked-out blocks are zero); no bias."""
    K, N = (1280, 5120) if layer == "fc1" else (5120, 1280)
    s = seed + (0 if layer == "fc1" else 100)
    crow, col = bsr_pattern(N // bs, K // bs, keep, s + 3)
    w = normal_f32((N, K), 0.02, s + 1)
    w[~block_mask_dense(N, K, crow, col, bs)] = 0.0
    d = dict(name=f"ViT-H {layer} BSR M={M} K={K} N={N} keep={keep}",
             w=w, crow=crow, col=col, K=K, N=N, M=M)
    if with_x:
        d["x"] = normal_bf16((M, K), 1.0, s)
    return d


def quant_sweep(seed: int = 0, M: int = 16384, K: int = 8192):
    return dict(name=f"quantize X [{M}, {K}]", x=normal_bf16((M, K), 1.0, seed))


def small_m(seed: int = 0, M: int = 16, K: int = 8192, N: int = 28672):
    return dict(name=f"small-M dense M={M} K={K} N={N}",
                x=normal_bf16((M, K), 1.0, seed), w=normal_f32((N, K), 0.02, seed + 1),
                bias=None)


def hqq(seed: int = 0, M: int = 16, N: int = 4096, K: int = 4096, group: int = 128,
        signed: bool = False):
    """Weight-only int4 linear, the HQQ benchmark shapes (N = K = 4096, group
    128, M from 16 to 1024): X bf16 [M, K] ~ N(0, 1); int4 codes int8 [N, K]
    uniform over 0..15 (u4) or -8..7 (s4); per (channel, group) bf16 scales
    uniform in [0.002, 0.02] and bf16 zero points uniform in [6, 9] (u4) or
    [-1.5, 1.5] (s4), non-integer like HQQ's optimised zero points.  Codes
    are unpacked: packing is part of the method.  Sub-seeds: X = seed, codes =
    seed+1, scales = seed+5, zero points = seed+6."""
    lo, hi = (-8, 7) if signed else (0, 15)
    zlo, zhi = (-1.5, 1.5) if signed else (6.0, 9.0)
    G = K // group
    return dict(name=f"HQQ int4 linear M={M} N={N} K={K} group={group}{' s4' if signed else ''}",
                x=normal_bf16((M, K), 1.0, seed),
                codes=uniform_int8((N, K), lo, hi, seed + 1),
                scale=f32_to_bf16_bits(uniform_f32((N, G), 0.002, 0.02, seed + 5)),
                zero=f32_to_bf16_bits(uniform_f32((N, G), zlo, zhi, seed + 6)),
                group=group, signed=signed)


def s24_mask(N: int, K: int, seed: int) -> np.ndarray:
    """bool [N, K]: in every group of four consecutive in-features exactly
    two kept positions, each of the six pairs equally likely."""
    pairs = np.array([[0, 1], [0, 2], [0, 3], [1, 2], [1, 3], [2, 3]], np.int64)
    choice = rng(seed).integers(0, 6, size=(N, K // 4))
    mask = np.zeros((N, K // 4, 4), bool)
    sel = pairs[choice]                                   # [N, K/4, 2]
    np.put_along_axis(mask, sel, True, axis=2)
    return mask.reshape(N, K)


def s24(seed: int = 0, M: int = 2048, K: int = 4096, N: int = 4096):
    """2:4-sparse linear: X bf16 [M, K] ~ N(0, 1); W fp32 [N, K] ~ N(0, 0.02)
    zeroed outside a uniform 2:4 mask (seed+3)."""
    w = normal_f32((N, K), 0.02, seed + 1)
    w[~s24_mask(N, K, seed + 3)] = 0.0
    return dict(name=f"2:4 sparse linear M={M} K={K} N={N}", x=normal_bf16((M, K), 1.0, seed), w=w)

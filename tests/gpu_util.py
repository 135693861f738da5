"""Helpers for the GPU parity tests: numpy <-> torch moves and the bf16 ulp
distance used as the tolerance (at most 1 bf16 ulp; ulp distance is taken on
the ordered bit patterns, with +0 and -0 equal)."""
import numpy as np
import torch


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _ordered(h: np.ndarray) -> np.ndarray:
    h = h.astype(np.int64)
    mag = h & 0x7FFF
    return np.where(h & 0x8000, -mag, mag)


def bf16_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.abs(_ordered(a) - _ordered(b))


def assert_bf16_close(got: np.ndarray, want: np.ndarray, max_ulp: int = 1):
    assert got.shape == want.shape
    d = bf16_ulp_diff(got, want)
    worst = int(d.max()) if d.size else 0
    assert worst <= max_ulp, f"max bf16 ulp diff {worst} at {np.unravel_index(int(d.argmax()), d.shape)}"
    return int((d != 0).sum())


def sample_rows(M: int, n_random: int, seed: int = 0) -> np.ndarray:
    fixed = [0, 1, 2, 63, 64, 127, 128, 129, 255, 256, M // 2, M - 129, M - 128, M - 127, M - 2, M - 1]
    r = np.random.Generator(np.random.Philox(key=seed)).choice(M, size=min(M, n_random), replace=False)
    rows = np.unique(np.clip(np.concatenate([np.array(fixed), r]), 0, M - 1))
    return rows.astype(np.int64)

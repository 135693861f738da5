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


def tile_rows(M: int, total: int = 1024, seed: int = 0, tile: int = 128) -> np.ndarray:
    """Rows for full-size parity: the first and last row of every `tile`-row
    block (so every M-tile of the 1-SM kernels and, with tile = 128, both
    halves of every 256-row pair tile), the rows around the middle, plus
    seeded random rows until at least `total` rows (or all M) are chosen."""
    starts = np.arange(0, M, tile)
    edges = np.concatenate([starts, np.minimum(starts + tile - 1, M - 1), [M // 2, M - 1]])
    rows = np.unique(np.clip(edges, 0, M - 1))
    if rows.size < min(total, M):
        rng = np.random.Generator(np.random.Philox(key=seed))
        rest = np.setdiff1d(np.arange(M), rows)
        extra = rng.choice(rest, size=min(total, M) - rows.size, replace=False)
        rows = np.unique(np.concatenate([rows, extra]))
    return rows.astype(np.int64)


def tile_cols(N: int, widths=(128, 224, 256), extra_step: int = 97) -> np.ndarray:
    """Output channels at both edges of every tile of each width (the swap
    arrangement's 128-channel tiles, the few-token dense arrangement's
    224-wide tiles, the 256-wide tiles), plus a regular stride through N."""
    cols = [np.arange(0, N, extra_step), [N - 1]]
    for w in widths:
        s = np.arange(0, N, w)
        cols += [s, np.minimum(s + w - 1, N - 1)]
    return np.unique(np.concatenate(cols)).astype(np.int64)

"""Pins for the oracle's 2:4 semi-structured sparse weight routines, checked
against things other than the oracle itself: a hand-worked example
(tests/golden/s24_worked_1x16.json), the format's invariants on random 2:4
weights, the rule for groups with fewer than two nonzeros, and numpy int64
matmuls of the decompressed weight."""
import json
import os

import numpy as np

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "s24_worked_1x16.json")


def test_worked_example():
    g = json.load(open(GOLD))
    W = np.array(g["W"], np.int8)
    v, m, bad = oracle.s24_compress(W)
    assert bad == 0
    assert v.tolist() == g["values"] and m.tolist() == g["meta"]
    assert np.array_equal(oracle.s24_decompress(v, m), W)
    x = np.array(g["x"], np.int8)
    assert oracle.gemm_s32(x, oracle.s24_decompress(v, m)).tolist() == g["acc"]


def _random_s24(N, K, seed):
    r = np.random.default_rng(seed)
    W = r.integers(-127, 128, size=(N, K)).astype(np.int8)
    W[~synth.s24_mask(N, K, seed)] = 0
    return W


def test_roundtrip_and_format_invariants():
    W = _random_s24(37, 256, 1)
    v, m, bad = oracle.s24_compress(W)
    assert bad == 0
    assert np.array_equal(oracle.s24_decompress(v, m), W)
    nib = np.stack([m & 0x0F, m >> 4], axis=2).reshape(37, 64)
    p0, p1 = nib & 3, nib >> 2
    assert (p0 < p1).all()
    # the kept values are the group's nonzeros, in position order
    groups = W.reshape(37, 64, 4)
    kept = np.stack([np.take_along_axis(groups, p0[..., None], 2)[..., 0],
                     np.take_along_axis(groups, p1[..., None], 2)[..., 0]], axis=2).reshape(37, 128)
    assert np.array_equal(kept, v)
    assert (np.count_nonzero(groups, axis=2) == np.count_nonzero(v.reshape(37, 64, 2), axis=2)).all()


def test_sparse_groups_fill_lowest_free_positions():
    W = np.zeros((1, 16), np.int8)
    W[0, 4 + 2] = 9          # one nonzero at position 2 -> kept positions (0, 2)
    W[0, 8 + 0] = -4         # one nonzero at position 0 -> (0, 1)
    v, m, _ = oracle.s24_compress(W)
    assert m[0, 0] == (0x4 | ((0 | (2 << 2)) << 4))      # group 0 empty -> (0, 1); group 1 -> (0, 2)
    assert m[0, 1] == (0x4 | (0x4 << 4))                  # group 2 -> (0, 1); group 3 empty -> (0, 1)
    assert v[0].tolist() == [0, 0, 0, 9, -4, 0, 0, 0]


def test_more_than_two_nonzeros_is_reported():
    W = np.zeros((2, 8), np.int8)
    W[1, 0:3] = [1, 2, 3]
    _, _, bad = oracle.s24_compress(W)
    assert bad == 1


def test_sparse_product_is_the_dense_product():
    r = np.random.default_rng(5)
    W = _random_s24(48, 512, 7)
    A = r.integers(-127, 128, size=(33, 512)).astype(np.int8)
    v, m, _ = oracle.s24_compress(W)
    acc = oracle.gemm_s32(A, oracle.s24_decompress(v, m))
    assert np.array_equal(acc.astype(np.int64), A.astype(np.int64) @ W.astype(np.int64).T)


def test_synth_mask_is_two_of_four():
    mk = synth.s24_mask(64, 256, 3)
    assert (mk.reshape(64, 64, 4).sum(axis=2) == 2).all()

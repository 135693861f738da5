"""Pins for the oracle's weight-only int4 (HQQ) routines, checked against
things other than the oracle itself:

* a worked example by hand (tests/golden/hqq_worked_2x4.json);
* hand-worked bf16 ties of the two rounding steps, and brute-force nearest-
  even rounding over exact rationals;
* PyTorch's CPU bf16 tensor arithmetic (q - z, then * s), whose single
  roundings are exact here because q - z and a bf16 product fit in fp32;
* numpy float64 matmuls for the forward and transposed products, and a
  one-hot activation that reads back a single dequantized weight;
* closed forms: s = 1, z = 0 gives the codes; integer z with a power-of-two
  s is exact; a group's scale moves only that group's columns.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hqq_worked_2x4.json")


def _bits(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def _vals(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits, np.uint16)).astype(np.float64)


def test_worked_example():
    g = json.load(open(GOLD))
    codes = np.array(g["codes"], np.int8)
    packed = oracle.hqq_pack(codes)
    assert packed.tolist() == g["packed"]
    assert np.array_equal(oracle.hqq_unpack(packed), codes)
    w = oracle.hqq_dequant(packed, _bits(g["scale"]), _bits(g["zero"]), g["group"])
    assert _vals(w).tolist() == g["w"]
    out = oracle.hqq_linear_f64(_bits(g["x"]), w)
    assert out.tolist() == g["out"]
    out_t = oracle.hqq_linear_t_f64(_bits(g["y"]), w)
    assert out_t.tolist() == g["out_t"]


def test_pack_nibble_order_and_signed_roundtrip():
    # u4: low nibble = even column, high nibble = odd column
    assert oracle.hqq_pack(np.array([[1, 2, 15, 0]], np.int8)).tolist() == [[0x21, 0x0F]]
    # s4: two's-complement nibbles
    s4 = np.array([[-1, 7, -8, 0]], np.int8)
    assert oracle.hqq_pack(s4).tolist() == [[0x7F, 0x08]]
    assert np.array_equal(oracle.hqq_unpack(oracle.hqq_pack(s4), signed=True), s4)
    r = np.random.default_rng(3)
    for lo, hi, sg in ((0, 15, False), (-8, 7, True)):
        c = r.integers(lo, hi + 1, size=(7, 40)).astype(np.int8)
        assert np.array_equal(oracle.hqq_unpack(oracle.hqq_pack(c), signed=sg), c)


def _nearest_even_bf16(v: Fraction) -> float:
    """Brute force: the bf16 value nearest to v, ties to even mantissa."""
    f = float(v)
    base = int(_bits([f])[0])
    best = None
    for b in range(max(base - 3, 0), base + 4):
        c = Fraction(float(_vals([b])[0]))
        d = abs(c - v)
        key = (d, b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return float(_vals([best[1]])[0])


def test_bf16_rounding_ties_and_brute_force():
    # (q=3, z=0.5, s=bf16(0.3)=0.30078125): 2.5 * 0.30078125 = 0.751953125, a tie -> 0.75
    assert oracle.double_to_bf16(0.751953125) == 0x3F40
    # 15 - 2^-5 = 14.96875 is a tie between 14.9375 and 15 -> 15 (even)
    assert oracle.double_to_bf16(14.96875) == 0x4170
    # 15 - 0.09375 = 14.90625 is a tie between 14.875 and 14.9375 -> 14.875 (even)
    assert oracle.double_to_bf16(14.90625) == 0x416E
    r = np.random.default_rng(11)
    for _ in range(300):
        v = Fraction(float(r.standard_normal() * 2.0 ** r.integers(-20, 20)))
        got = float(_vals([oracle.double_to_bf16(float(v))])[0])
        assert got == _nearest_even_bf16(v)


@pytest.mark.parametrize("signed", [False, True])
@pytest.mark.parametrize("group", [32, 64, 128])
def test_dequant_matches_torch_bf16_arithmetic(signed, group):
    d = synth.hqq(seed=5, M=1, N=24, K=256, group=group, signed=signed)
    packed = oracle.hqq_pack(d["codes"])
    w = oracle.hqq_dequant(packed, d["scale"], d["zero"], group, signed=signed)
    q = torch.from_numpy(d["codes"].astype(np.float32)).to(torch.bfloat16)
    z = torch.from_numpy(_vals(d["zero"]).astype(np.float32)).to(torch.bfloat16)
    s = torch.from_numpy(_vals(d["scale"]).astype(np.float32)).to(torch.bfloat16)
    z = z.repeat_interleave(group, dim=1)
    s = s.repeat_interleave(group, dim=1)
    ref = ((q - z) * s).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(w, ref)


def test_dequant_closed_forms():
    r = np.random.default_rng(2)
    for signed, lo, hi in ((False, 0, 15), (True, -8, 7)):
        c = r.integers(lo, hi + 1, size=(5, 64)).astype(np.int8)
        p = oracle.hqq_pack(c)
        one = _bits(np.ones((5, 2)))
        zero = _bits(np.zeros((5, 2)))
        assert np.array_equal(_vals(oracle.hqq_dequant(p, one, zero, 32, signed)), c.astype(np.float64))
        zi = r.integers(-3, 12, size=(5, 2)).astype(np.float32)
        s = np.float32(2.0 ** -4)
        w = _vals(oracle.hqq_dequant(p, _bits(np.full((5, 2), s)), _bits(zi), 32, signed))
        exp = (c.astype(np.float64) - np.repeat(zi, 32, axis=1)) * float(s)
        assert np.array_equal(w, exp)


def test_group_scale_moves_only_its_columns():
    d = synth.hqq(seed=8, M=1, N=4, K=256, group=64)
    p = oracle.hqq_pack(d["codes"])
    w0 = oracle.hqq_dequant(p, d["scale"], d["zero"], 64)
    sc = d["scale"].copy()
    sc[2, 1] = _bits([0.5])[0]
    w1 = oracle.hqq_dequant(p, sc, d["zero"], 64)
    diff = w0 != w1
    assert diff[2, 64:128].any()
    diff[2, 64:128] = False
    assert not diff.any()


@pytest.mark.parametrize("M,N,K", [(3, 5, 64), (9, 17, 96)])
def test_products_match_numpy(M, N, K):
    d = synth.hqq(seed=M, M=M, N=N, K=K, group=32)
    w = oracle.hqq_dequant(oracle.hqq_pack(d["codes"]), d["scale"], d["zero"], 32)
    x = _vals(d["x"])
    wv = _vals(w)
    out = oracle.hqq_linear_f64(d["x"], w)
    assert np.allclose(out, x @ wv.T, rtol=1e-13, atol=1e-13)
    y = synth.normal_bf16((M, N), 1.0, 77)
    out_t = oracle.hqq_linear_t_f64(y, w)
    assert out_t.shape == (M, K)
    assert np.allclose(out_t, _vals(y) @ wv, rtol=1e-13, atol=1e-13)


def test_one_hot_activation_reads_one_weight():
    d = synth.hqq(seed=4, M=1, N=6, K=64, group=32)
    w = oracle.hqq_dequant(oracle.hqq_pack(d["codes"]), d["scale"], d["zero"], 32)
    for k in (0, 1, 31, 32, 63):
        x = np.zeros((1, 64), np.float32)
        x[0, k] = 1.0
        out = oracle.hqq_linear_f64(_bits(x), w)
        assert np.array_equal(out[0], _vals(w)[:, k])

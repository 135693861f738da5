"""Pins for the CPU oracle: it is checked against the mathematics, never
against itself.

* hand-worked 4x4 example (tests/golden/worked_4x4.json), itself re-derived
  here in exact rational arithmetic;
* exact brute force (tests/exact.py) for quantization and the epilogue;
* numpy's int64 matmul and the oracle's own int64 twin for the int8 GEMM;
* closed forms (constant operands, identity weight, the int32 overflow bound
  of the "int8 dynamic quant + bsr support" review: 2^31 / 2^14);
* invariants (absmax element -> +-127, |x - q s| <= s/2, BSR == dense on the
  densified weight, "no bias" is not "+0 bias").
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import exact
import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "worked_4x4.json")


def _gold():
    with open(GOLD) as f:
        return json.load(f)


def _bits(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def _vals(bits):
    return synth.bf16_bits_to_f32(bits)


# ---------------------------------------------------------------- worked example

def test_worked_example_exact_rederivation():
    g = _gold()
    xb = _bits(g["x"])
    for i, row in enumerate(xb):
        q, s = exact.quantize_row_exact([exact.bf16_value(h) for h in row])
        assert q == g["q"][i]
        assert float(s) == g["s_row"][i]
    for n, row in enumerate(g["w"]):
        q, s = exact.quantize_row_exact([Fraction(v) for v in row])
        assert q == g["w_q"][n]
        assert float(s) == g["s_col"][n]
    acc = np.array(g["q"], np.int64) @ np.array(g["w_q"], np.int64).T
    assert acc.tolist() == g["acc"]
    bb = _bits(g["bias"])
    for m in range(4):
        for n in range(4):
            h = exact.epilogue_exact(g["acc"][m][n], np.float32(g["s_row"][m]),
                                     np.float32(g["s_col"][n]), int(bb[n]))
            assert float(exact.bf16_value(h)) == g["out"][m][n]


def test_worked_example_oracle():
    g = _gold()
    q, s = oracle.quantize_rows_bf16(_bits(g["x"]))
    assert q.tolist() == g["q"]
    assert s.tolist() == [np.float32(v) for v in g["s_row"]]
    wq, sc = oracle.quantize_rows_f32(np.array(g["w"], np.float32))
    assert wq.tolist() == g["w_q"]
    assert sc.tolist() == [np.float32(v) for v in g["s_col"]]
    acc = oracle.gemm_s32(q, wq)
    assert acc.tolist() == g["acc"]
    out = oracle.epilogue_bf16(acc, s, sc, _bits(g["bias"]))
    assert _vals(out).tolist() == g["out"]


def test_near_tie_row():
    g = _gold()["near_tie_row"]
    q, _ = oracle.quantize_rows_bf16(_bits([g["x"]]))
    assert q[0].tolist() == g["q"]


# ---------------------------------------------------------------- quantization

def test_quantize_brute_force_random():
    x = synth.normal_bf16((6, 48), 1.0, 11)
    x[1] = synth.normal_bf16((48,), 1e-3, 12)          # small magnitudes
    x[2, 7] = _bits([300.0])[0]                           # one outlier
    x[3] = _bits(np.zeros(48))                            # all-zero row
    x[4] = synth.normal_bf16((48,), 1e-9, 13)            # absmax below eps
    q, s = oracle.quantize_rows_bf16(x)
    for i in range(x.shape[0]):
        qe, se = exact.quantize_row_exact([exact.bf16_value(h) for h in x[i]])
        assert q[i].tolist() == qe
        assert s[i] == se


def test_quantize_f32_brute_force_random():
    w = synth.normal_f32((5, 40), 0.02, 21)
    q, s = oracle.quantize_rows_f32(w)
    for i in range(w.shape[0]):
        qe, se = exact.quantize_row_exact([Fraction(float(v)) for v in w[i]])
        assert q[i].tolist() == qe
        assert s[i] == se


def test_quantize_exact_ties_go_to_even():
    # absmax 127 -> scale exactly 1.0, so x/s = x and every .5 is a true tie.
    row = [127.0, 2.5, -0.5, 0.5, 1.5, 63.5, -63.5, 126.5, -126.5, 3.5]
    q, s = oracle.quantize_rows_bf16(_bits([row]))
    assert s[0] == np.float32(1.0)
    assert q[0].tolist() == [127, 2, 0, 0, 2, 64, -64, 126, -126, 4]


def test_quantize_invariants_tiny_config():
    d = synth.tiny(0)
    q, s = oracle.quantize_rows_bf16(d["x"])
    xv = _vals(d["x"]).astype(np.float64)
    absmax = np.abs(xv).max(axis=1)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    for i in range(q.shape[0]):
        j = int(np.argmax(np.abs(xv[i])))
        assert abs(int(q[i, j])) == 127
        assert np.sign(q[i, j]) == np.sign(xv[i, j])
    # |x/s - fl32(x/s)| <= half an fp32 ulp below 128 = 2^-18, so
    # |x - q s| <= s (1/2 + 2^-18) = s/2 (1 + 2^-17); fl32(x/s) can land on a
    # tie the exact ratio does not reach (e.g. -63.4999982 -> -63.5 -> -64).
    err = np.abs(xv - q.astype(np.float64) * s[:, None].astype(np.float64))
    assert np.all(err <= s[:, None] / 2 * (1 + 2.0 ** -17))
    # the scale itself: s = fp32(absmax / 127), within half an fp32 ulp
    assert np.all(np.abs(s.astype(np.float64) - absmax / 127) <= np.spacing(s) / 2)


def test_quantize_zero_and_tiny_rows():
    x = np.zeros((2, 16), np.uint16)
    x[1] = _bits(np.full(16, 1e-9))
    q, s = oracle.quantize_rows_bf16(x)
    eps_scale = exact.fl32(Fraction(float(exact.EPS)) / 127)
    assert s[0] == eps_scale and s[1] == eps_scale
    assert q[0].tolist() == [0] * 16
    # 1e-9 (as bf16) / (1e-8/127) ~ 12.7 -> 13: not exempt from rounding, only
    # from the "absmax maps to 127" invariant
    qe, _ = exact.quantize_row_exact([exact.bf16_value(h) for h in x[1]])
    assert q[1].tolist() == qe


# ---------------------------------------------------------------- GEMM

def test_gemm_matches_numpy_int64_and_twin():
    A = synth.uniform_int8((17, 96), -127, 127, 31)
    W = synth.uniform_int8((13, 96), -127, 127, 32)
    acc = oracle.gemm_s32(A, W)
    ref = A.astype(np.int64) @ W.astype(np.int64).T
    assert np.array_equal(acc.astype(np.int64), ref)
    assert np.array_equal(oracle.gemm_s64(A, W), ref)
    # square case: A @ W^T must differ from A @ W (a transposed operand)
    S = synth.uniform_int8((32, 32), -127, 127, 33)
    acc_sq = oracle.gemm_s32(S, S[::-1].copy())
    assert np.array_equal(acc_sq.astype(np.int64), S.astype(np.int64) @ S[::-1].astype(np.int64).T)
    assert not np.array_equal(acc_sq.astype(np.int64), S.astype(np.int64) @ S[::-1].astype(np.int64))


def test_gemm_closed_form_constants():
    K = 1000
    A = np.full((3, K), 127, np.int8)
    W = np.full((2, K), -127, np.int8)
    W[1] = 1
    acc = oracle.gemm_s32(A, W)
    assert acc[:, 0].tolist() == [-K * 127 * 127] * 3
    assert acc[:, 1].tolist() == [K * 127] * 3


def test_int32_overflow_bound():
    # |acc| <= K * 127^2 fits int32 iff K <= floor((2^31 - 1) / 127^2) = 133144
    kmax = (2 ** 31 - 1) // (127 * 127)
    assert kmax == 133144
    for K, fits in ((kmax, True), (kmax + 1, False)):
        A = np.full((1, K), 127, np.int8)
        W = np.full((1, K), 127, np.int8)
        a32 = int(oracle.gemm_s32(A, W)[0, 0])
        a64 = int(oracle.gemm_s64(A, W)[0, 0])
        assert a64 == K * 127 * 127
        assert (a32 == a64) == fits


def test_identity_weight_returns_quantized_activations():
    K = 64
    x = synth.normal_bf16((9, K), 1.0, 41)
    q, _ = oracle.quantize_rows_bf16(x)
    wq, sc = oracle.quantize_rows_f32(np.eye(K, dtype=np.float32))
    assert np.array_equal(wq, 127 * np.eye(K, dtype=np.int8))
    assert np.all(sc == exact.fl32(Fraction(1, 127)))
    acc = oracle.gemm_s32(q, wq)
    assert np.array_equal(acc, 127 * q.astype(np.int32))


# ---------------------------------------------------------------- epilogue

def test_epilogue_brute_force():
    r = synth.rng(51)
    acc = r.integers(-2 ** 31 // 2, 2 ** 31 // 2, size=(5, 7)).astype(np.int32)
    acc[0, :3] = [0, 1, -1]
    acc[1, :2] = [16777217, -16777219]       # int -> fp32 must round
    s_row = synth.uniform_f32((5,), 0.001, 0.05, 52)
    s_col = synth.uniform_f32((7,), 0.001, 0.05, 53)
    bias = synth.normal_bf16((7,), 0.1, 54)
    for b in (None, bias):
        out = oracle.epilogue_bf16(acc, s_row, s_col, b)
        for m in range(5):
            for n in range(7):
                e = exact.epilogue_exact(int(acc[m, n]), s_row[m], s_col[n],
                                         None if b is None else int(b[n]))
                assert int(out[m, n]) == e, (m, n)


def test_epilogue_no_bias_is_not_zero_bias():
    acc = np.array([[-1]], np.int32)
    s = np.array([1e-30], np.float32)
    out_none = oracle.epilogue_bf16(acc, s, s, None)
    out_zero = oracle.epilogue_bf16(acc, s, s, np.zeros(1, np.uint16))
    assert int(out_none[0, 0]) == 0x8000        # -0.0 survives with no addition
    assert int(out_zero[0, 0]) == 0x0000        # -0.0 + 0.0 = +0.0


def test_epilogue_left_to_right_order_matters():
    # (acc * s_row) * s_col differs from acc * (s_row * s_col) for these values;
    # the oracle must take the first reading.
    acc = np.array([[-311612264]], np.int32)
    s_row = np.array([0.033129707], np.float32)
    s_col = np.array([0.039576802], np.float32)
    out = oracle.epilogue_bf16(acc, s_row, s_col)
    left = exact.epilogue_exact(-311612264, s_row[0], s_col[0])
    both = exact.fl32(Fraction(float(s_row[0])) * Fraction(float(s_col[0])))
    right = exact.bf16(Fraction(float(exact.fl32(Fraction(float(exact.fl32(Fraction(-311612264))))
                                                 * Fraction(float(both))))))
    assert left != right
    assert int(out[0, 0]) == left


# ---------------------------------------------------------------- BSR

def _np_densify(N, K, crow, col, values, bs):
    W = np.zeros((N, K), np.int32)
    for b in range(N // bs):
        for p in range(crow[b], crow[b + 1]):
            W[b * bs:(b + 1) * bs, col[p] * bs:(col[p] + 1) * bs] += values[p]
    return W


@pytest.mark.parametrize("bs", [64, 32, 16])
def test_bsr_equals_dense_on_densified_weight(bs):
    N, K, M = 5 * bs, 4 * bs, 37
    crow, col = synth.bsr_pattern(N // bs, K // bs, 0.3, 61)
    crow[2:] = np.maximum(crow[2:], crow[2])       # keep it canonical
    assert crow[-1] == len(col)
    values = synth.uniform_int8((len(col), bs, bs), -127, 127, 62)
    A = synth.uniform_int8((M, K), -127, 127, 63)
    acc = oracle.bsr_gemm_s32(A, N, crow, col, values, bs)
    Wd = _np_densify(N, K, crow, col, values, bs)
    assert np.array_equal(oracle.bsr_densify(N, K, crow, col, values, bs), Wd)
    ref = A.astype(np.int64) @ Wd.astype(np.int64).T
    assert np.array_equal(acc.astype(np.int64), ref)
    empty = [b for b in range(N // bs) if crow[b] == crow[b + 1]]
    for b in empty:
        assert not acc[:, b * bs:(b + 1) * bs].any()


def test_bsr_pack_roundtrip_and_masked_quantization():
    d = synth.vit_h_bsr(0, "fc1", M=8, keep=0.1, with_x=False)
    wq, sc = oracle.quantize_rows_f32(d["w"])
    mask = synth.block_mask_dense(d["N"], d["K"], d["crow"], d["col"])
    assert not wq[~mask].any()                     # masked blocks stay 0
    vals = oracle.bsr_pack(wq, d["crow"], d["col"])
    assert vals.shape == (160, 64, 64)
    assert np.array_equal(_np_densify(d["N"], d["K"], d["crow"], d["col"], vals, 64), wq)


def test_bsr_duplicate_blocks_add():
    bs = 64
    crow = np.array([0, 2], np.int32)
    col = np.array([1, 1], np.int32)
    values = synth.uniform_int8((2, bs, bs), -127, 127, 71)
    A = synth.uniform_int8((3, 2 * bs), -127, 127, 72)
    acc = oracle.bsr_gemm_s32(A, bs, crow, col, values, bs)
    ref = A[:, bs:].astype(np.int64) @ (values[0].astype(np.int64) + values[1]).T
    assert np.array_equal(acc.astype(np.int64), ref)


# ---------------------------------------------------------------- accuracy

def _rel_frob(x_bits, w, out_bits, bias_bits=None):
    ref = _vals(x_bits).astype(np.float64) @ w.astype(np.float64).T
    if bias_bits is not None:
        ref = ref + _vals(bias_bits).astype(np.float64)
    got = _vals(out_bits).astype(np.float64)
    return np.linalg.norm(got - ref) / np.linalg.norm(ref)


def test_frobenius_gate_tiny():
    d = synth.tiny(0)
    wq, sc = oracle.quantize_rows_f32(d["w"])
    out, _, _ = oracle.dynamic_linear_bf16(d["x"], wq, sc, d["bias"])
    assert _rel_frob(d["x"], d["w"], out, d["bias"]) <= 2e-2


@pytest.mark.slow
def test_frobenius_llm_outliers_reported_not_gated():
    # 1% of channels x20: per-token int8 alone gives ~5e-2 relative error here;
    # without the outliers the same arithmetic meets 2e-2.
    d = synth.llm(0, M=64)
    wq, sc = oracle.quantize_rows_f32(d["w"])
    out, _, _ = oracle.dynamic_linear_bf16(d["x"], wq, sc)
    e = _rel_frob(d["x"], d["w"], out)
    assert 3e-2 < e < 8e-2
    d2 = synth.small_m(0, M=64, K=4096, N=512)
    wq2, sc2 = oracle.quantize_rows_f32(d2["w"])
    out2, _, _ = oracle.dynamic_linear_bf16(d2["x"], wq2, sc2)
    assert _rel_frob(d2["x"], d2["w"], out2) <= 2e-2


# ---------------------------------------------------------------- FP8 (e4m3)
# The sibling precision of the vLLM csrc/quantization commits (dynamic scales,
# scaled values clamped to the e4m3 range): s = fp32(max(absmax, 1e-8)/448),
# q = e4m3(clamp(fp32(x/s), -448, 448)), round to nearest even.

def _e4m3_values_from_definition():
    """All 256 codes decoded from the format's definition (1-4-3, bias 7,
    e = 15 & m = 7 is NaN, exponent 0 subnormal), written independently."""
    vals = []
    for c in range(256):
        sgn = -1.0 if c & 0x80 else 1.0
        e, m = (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            vals.append(np.nan)
        elif e == 0:
            vals.append(sgn * m * 2.0 ** -9)
        else:
            vals.append(sgn * (8 + m) * 2.0 ** (e - 10))
    return np.array(vals)


def test_e4m3_decode_table():
    got = oracle.e4m3_to_float64(np.arange(256))
    want = _e4m3_values_from_definition()
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x38] == 1.0
    pos = got[:0x7F]
    assert np.all(np.diff(pos) > 0)            # codes 0 .. 0x7E increase


def test_e4m3_rounding_is_nearest_even_by_brute_force():
    table = _e4m3_values_from_definition()[:0x7F]          # non-negative finite values
    rng = np.random.default_rng(5)
    mids = (table[1:] + table[:-1]) / 2                    # every tie
    xs = np.concatenate([rng.uniform(0, 460, 3000), rng.uniform(0, 0.03, 3000), table, mids,
                         np.nextafter(mids.astype(np.float32), np.float32(0)),
                         np.nextafter(mids.astype(np.float32), np.float32(1e9))]).astype(np.float32)
    got = oracle.float_to_e4m3(xs)
    for x, c in zip(xs.astype(np.float64), got):
        if x >= 448.0:
            assert c == 0x7E
            continue
        d = np.abs(table - x)
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert c == want, (x, c, want)
    assert np.array_equal(oracle.float_to_e4m3(-xs[:500]), got[:500] | 0x80)


def test_fp8_quantize_matches_definition_and_invariants():
    x = synth.normal_bf16((33, 300), 1.0, 77)
    x[0] = 0
    q, s = oracle.quantize_rows_bf16_fp8(x)
    xf = synth.bf16_bits_to_f32(x) if hasattr(synth, "bf16_bits_to_f32") else \
        (x.astype(np.uint32) << 16).view(np.float32)
    a = np.abs(xf).max(axis=1)
    s_want = (np.maximum(a, np.float32(1e-8)) / np.float32(448)).astype(np.float32)
    assert np.array_equal(s.view(np.uint32), s_want.view(np.uint32))
    ratio = np.clip((xf / s_want[:, None]).astype(np.float32), -448, 448)
    table = _e4m3_values_from_definition()
    vals = table[q]
    # each code is the e4m3 value nearest the IEEE quotient (ties checked above)
    fin = table[:0x7F]
    for i in range(1, 33):
        for k in range(0, 300, 7):
            r = float(abs(ratio[i, k]))
            assert abs(abs(vals[i, k]) - r) == np.abs(fin - r).min()
    # the absmax element maps to +-448 in every nonzero row
    for i in range(1, 33):
        j = int(np.argmax(np.abs(xf[i])))
        assert q[i, j] & 0x7F == 0x7E
    assert not q[0].any()


def test_fp8_gemm_is_the_exact_sum():
    rng = np.random.default_rng(8)
    A = rng.integers(0, 256, (9, 96)).astype(np.uint8)
    W = rng.integers(0, 256, (7, 96)).astype(np.uint8)
    A[(A & 0x7F) == 0x7F] = 0x12                 # no NaN codes
    W[(W & 0x7F) == 0x7F] = 0x35
    Av, Wv = _e4m3_values_from_definition()[A], _e4m3_values_from_definition()[W]
    want = Av @ Wv.T
    got = oracle.gemm_fp8_f64(A, W)
    assert np.array_equal(got, want)
    # products of e4m3 values are exact in double: a transposed operand fails
    assert not np.array_equal(oracle.gemm_fp8_f64(A, W[::-1]), want)

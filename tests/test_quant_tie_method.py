"""The division-free rounding of the CUDA quantize kernels' bf16 path,
restated in numpy and checked exhaustively.

Per-token int8 quantization (pytorch/ao PR 821, "int8 dynamic quant + bsr
support"; Paddle PR 41770's absmax / 127 scale) rounds fp32(x / s) to the
nearest integer, ties to even.  For bf16 activations the kernels form the
correctly rounded quotient without a division, by Markstein's correction step
(P. Markstein, IBM J. Res. Dev. 34(1), 1990):

    q0 = fp32(x * inv)            inv = fp32(1 / s)
    r  = fp32(x - q0 * s)         (one fma)
    q1 = fp32(q0 + r * inv)       (one fma)

and round q1 with the 1.5 * 2^23 addition.  This test restates those three
steps exactly (float64 products, which fit in 53 bits; an error-free sum for
the last fma; one rounding to float32 each) and checks, for every positive
bf16 absmax and every bf16 value x with |x| <= absmax, that rint(q1) equals
rint of numpy's IEEE float32 quotient.  q1 itself may differ from the IEEE
quotient only when the quotient is below 1/4 (r then underflows), where both
round to 0.
"""
import numpy as np
import pytest


def _two_sum(a, b):
    s = a + b
    bb = s - a
    return s, (a - (s - bb)) + (b - bb)


def _round32(hi, lo):
    """float32 rounding of the exact value hi + lo (|lo| <= ulp64(hi) / 2)."""
    f = hi.astype(np.float32)
    f64 = f.astype(np.float64)
    up = np.nextafter(f, np.float32(np.inf))
    dn = np.nextafter(f, np.float32(-np.inf))
    on_up = hi == (f64 + up.astype(np.float64)) / 2      # hi on a float32 midpoint: lo decides
    on_dn = hi == (f64 + dn.astype(np.float64)) / 2
    f = np.where(on_up & (lo > 0), up, f)
    f = np.where(on_dn & (lo < 0), dn, f)
    return f.astype(np.float32)


@pytest.mark.slow
def test_markstein_rounding_matches_ieee_division_for_all_bf16():
    v_all = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    v_all = v_all[np.isfinite(v_all)]
    checked = code_mismatch = big_quotient_mismatch = 0
    for a in v_all[v_all > 0]:
        s = np.float32(np.maximum(a, np.float32(1e-8)) / np.float32(127))
        inv = np.float32(np.float32(1) / s)
        x = v_all[np.abs(v_all) <= a]
        ref = (x / s).astype(np.float32)
        q0 = (x * inv).astype(np.float32)
        r = (x.astype(np.float64) - q0.astype(np.float64) * np.float64(s)).astype(np.float32)
        hi, lo = _two_sum(q0.astype(np.float64), r.astype(np.float64) * np.float64(inv))
        q1 = _round32(hi, lo)
        code_mismatch += int((np.rint(q1) != np.rint(ref)).sum())
        big_quotient_mismatch += int(((q1 != ref) & (np.abs(ref) >= 0.25)).sum())
        checked += x.size
    assert checked > 10 ** 9
    assert code_mismatch == 0
    assert big_quotient_mismatch == 0


def _e4m3_codes(x):
    """Vectorised round-to-nearest-even float -> e4m3 code, magnitudes clamped to 448."""
    x = np.asarray(x, np.float64)
    neg = np.signbit(x)
    a = np.minimum(np.abs(x), 448.0)
    sub = a < 2.0 ** -6
    m, e = np.frexp(np.where(sub, 1.0, a))
    ex = e - 1
    mq = np.rint((m * 2 - 1) * 8)
    ex = np.where(mq == 8, ex + 1, ex)
    mq = np.where(mq == 8, 0, mq)
    code = np.where(sub, np.rint(a * 2.0 ** 9), np.minimum((ex + 7) * 8 + mq, 0x7E))
    return (code.astype(np.uint16) | (neg.astype(np.uint16) << 7)).astype(np.uint8)


@pytest.mark.slow
def test_markstein_quotient_gives_ieee_e4m3_codes_for_all_bf16():
    """The FP8 path (s = absmax / 448) uses the same correction step; wherever
    its quotient differs from the IEEE one (always below 1/4, r underflowing)
    the e4m3 codes of the two agree, for every bf16 (absmax, x) pair."""
    v_all = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    v_all = v_all[np.isfinite(v_all)]
    differing = code_mismatch = 0
    for a in v_all[v_all > 0]:
        s = np.float32(np.maximum(a, np.float32(1e-8)) / np.float32(448))
        inv = np.float32(np.float32(1) / s)
        x = v_all[np.abs(v_all) <= a]
        ref = (x / s).astype(np.float32)
        q0 = (x * inv).astype(np.float32)
        r = (x.astype(np.float64) - q0.astype(np.float64) * np.float64(s)).astype(np.float32)
        hi, lo = _two_sum(q0.astype(np.float64), r.astype(np.float64) * np.float64(inv))
        q1 = _round32(hi, lo)
        mm = q1 != ref
        if mm.any():
            differing += int(mm.sum())
            assert np.all(np.abs(ref[mm]) < 0.25)
            code_mismatch += int((_e4m3_codes(q1[mm]) != _e4m3_codes(ref[mm])).sum())
    assert differing > 0          # the underflow cases exist ...
    assert code_mismatch == 0     # ... and never change a code

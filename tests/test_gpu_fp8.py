"""GPU parity of the dynamic FP8 (e4m3) sibling path against the CPU oracle.

Quantization (activations bf16 -> e4m3 per token, weights fp32 -> e4m3 per
channel) is bit-exact.  The product runs on the tensor cores with an fp32
accumulator (kind::f8f6f4): every product of two e4m3 values is exact in
fp32, but the order and precision of the hardware's sum are its own, so the
raw accumulators are compared with the oracle's exact (float64) sum within a
bound, and the bf16 outputs with the exact value within that bound plus one
bf16 rounding.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_bits, sample_rows, tile_rows, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

dq = pytest.importorskip("quantized_gemm_token_b200") if torch.cuda.is_available() else None

# |acc - exact| <= ACC_REL * sum_k |a_k w_k|: 2^-20, sixteen times the unit
# roundoff of fp32 (the sum of a K-term dot product rounded term by term in
# any order can be off by up to (K-1) * 2^-24 of that sum; the tensor core's
# blocked sum is measured far inside this bound).
ACC_REL = 2.0 ** -20


@pytest.fixture(autouse=True)
def _sync_and_check():
    yield
    if torch.cuda.is_available():
        assert dq.dq_sync_status() == dq.DQ_OK


def _bf16_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("M,K", [(1, 16), (3, 64), (64, 256), (7, 1280), (5, 4096), (9, 5120), (2, 8192),
                                 (300, 136), (4, 1000), (0, 64)])
def test_quantize_rows_fp8_bit_exact(M, K):
    x = synth.normal_bf16((max(M, 1), K), 1.0, 40 + K)[:M]
    if M >= 3:
        x[0] = 0
        x[1] = synth.normal_bf16((K,), 1e-9, 41)
        x[2] = synth.f32_to_bf16_bits(np.float32(4.0) * (np.arange(K) % 9 - 4).astype(np.float32))
    q, s = dq.dq_quantize_rows_fp8(to_dev_bf16(x))
    qo, so = oracle.quantize_rows_bf16_fp8(x)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


@pytest.mark.parametrize("a", [1.0, 448.0, 3.5, 0.0123, 3e-6, 1e-9, 65504.0, 1.5e30])
def test_quantize_fp8_every_bf16_pattern_below_absmax(a):
    """All bf16 values |x| <= a in one row whose absmax is a."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = _bf16_to_f32(bits)
    keep = np.isfinite(vals) & (np.abs(vals) <= np.float32(a))
    row = bits[keep]
    row = np.concatenate([row, synth.f32_to_bf16_bits(np.array([a], np.float32))])
    K = (len(row) + 15) // 16 * 16
    x = np.zeros((1, K), np.uint16)
    x[0, :len(row)] = row
    q, s = dq.dq_quantize_rows_fp8(to_dev_bf16(x))
    qo, so = oracle.quantize_rows_bf16_fp8(x)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


@pytest.mark.parametrize("N,K", [(256, 256), (5120, 1280), (33, 4096), (64, 100)])
def test_quantize_weight_fp8_bit_exact(N, K):
    w = synth.normal_f32((N, K), 0.02, 50 + K)
    w[0, :3] = [0.5, -0.25, 0.125]
    wq, sc = dq.dq_quantize_weight_fp8(to_dev(w))
    wo, so = oracle.quantize_rows_f32_fp8(w)
    assert np.array_equal(wq.cpu().numpy(), wo)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), so.view(np.uint32))


def _fp8_operands(M, N, K, seed):
    x = synth.normal_bf16((M, K), 1.0, seed)
    w = synth.normal_f32((N, K), 0.02, seed + 1)
    q, s = oracle.quantize_rows_bf16_fp8(x)
    wq, sc = oracle.quantize_rows_f32_fp8(w)
    return x, w, q, s, wq, sc


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (129, 264, 128), (300, 520, 384), (513, 1032, 4096),
                                   (2048, 4096, 512), (64, 8, 1280)])
def test_fp8_linear_against_the_exact_sum(M, N, K):
    x, w, q, s, wq, sc = _fp8_operands(M, N, K, 600 + M + N + K)
    bias = synth.normal_bf16((N,), 0.1, 7)
    qd, wd = to_dev(q), to_dev(wq)
    acc = dq.dq_fp8_linear(qd, None, wd, None, out_dtype="f32").cpu().numpy().astype(np.float64)
    out = dq.dq_fp8_linear(qd, to_dev(s), wd, to_dev(sc), bias=to_dev_bf16(bias))
    rows = tile_rows(M, total=256, seed=M)
    exact = oracle.gemm_fp8_f64(q[rows], wq)
    qa = np.abs(oracle.e4m3_to_float64(q[rows]))
    wa = np.abs(oracle.e4m3_to_float64(wq))
    mag = qa @ wa.T                                   # sum_k |a_k w_k|
    err = np.abs(acc[rows] - exact)
    assert np.all(err <= ACC_REL * mag + 1e-30)
    # bf16 out: the exact value through the epilogue's scaling, within the
    # accumulation bound (scaled) plus one bf16 rounding
    y = exact * s[rows, None].astype(np.float64) * sc[None, :].astype(np.float64) + \
        _bf16_to_f32(bias)[None, :].astype(np.float64)
    got = _bf16_to_f32(bf16_bits(out)[rows]).astype(np.float64)
    tol = ACC_REL * mag * s[rows, None] * sc[None, :] + np.abs(y) * 2.0 ** -8 + 1e-30
    assert np.all(np.abs(got - y) <= tol)


@pytest.mark.parametrize("M,N,K", [(300, 520, 384), (513, 1032, 4096), (1600, 4104, 2048)])
def test_fp8_pair_kernel_against_the_exact_sum(M, N, K):
    """The 2-SM pair kernel with e4m3 operands (forced with schedule 3;
    the automatic choice from 1536 tokens and K >= 2048): ragged rows,
    columns and both tile widths, within the same bounds as the 1-SM kernel."""
    x, w, q, s, wq, sc = _fp8_operands(M, N, K, 700 + M + N + K)
    qd, wd = to_dev(q), to_dev(wq)
    dq.dq_debug_set_schedule(3)
    try:
        acc = dq.dq_fp8_linear(qd, None, wd, None, out_dtype="f32").cpu().numpy().astype(np.float64)
        out = dq.dq_fp8_linear(qd, to_dev(s), wd, to_dev(sc))
    finally:
        dq.dq_debug_set_schedule(0)
    rows = tile_rows(M, total=256, seed=M)
    exact = oracle.gemm_fp8_f64(q[rows], wq)
    mag = np.abs(oracle.e4m3_to_float64(q[rows])) @ np.abs(oracle.e4m3_to_float64(wq)).T
    assert np.all(np.abs(acc[rows] - exact) <= ACC_REL * mag + 1e-30)
    y = exact * s[rows, None].astype(np.float64) * sc[None, :].astype(np.float64)
    got = _bf16_to_f32(bf16_bits(out)[rows]).astype(np.float64)
    assert np.all(np.abs(got - y) <= ACC_REL * mag * s[rows, None] * sc[None, :] + np.abs(y) * 2.0 ** -8 + 1e-30)


def test_fp8_llm_shaped_layer_and_accuracy():
    d = synth.llm(0)
    M, K, N = d["x"].shape[0], d["x"].shape[1], d["w"].shape[0]
    q, s = dq.dq_quantize_rows_fp8(to_dev_bf16(d["x"]))
    wq, sc = dq.dq_quantize_weight_fp8(to_dev(d["w"]))
    out = dq.dq_fp8_linear(q, s, wq, sc)
    qo_all, so_all = oracle.quantize_rows_bf16_fp8(d["x"])
    assert np.array_equal(q.cpu().numpy(), qo_all)            # every row's codes
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so_all.view(np.uint32))
    rows = tile_rows(M)                         # 1024 rows, both edges of all 16 M-tiles
    qo, so = qo_all[rows], so_all[rows]
    wo, sco = oracle.quantize_rows_f32_fp8(d["w"])
    assert np.array_equal(wq.cpu().numpy(), wo)
    exact = oracle.gemm_fp8_f64(qo, wo)
    mag = np.abs(oracle.e4m3_to_float64(qo)) @ np.abs(oracle.e4m3_to_float64(wo)).T
    y = exact * so[:, None].astype(np.float64) * sco[None, :].astype(np.float64)
    got = _bf16_to_f32(bf16_bits(out)[rows]).astype(np.float64)
    assert np.all(np.abs(got - y) <= ACC_REL * mag * so[:, None] * sco[None, :] + np.abs(y) * 2.0 ** -8 + 1e-30)
    # accuracy against the unquantized fp32 product (reported in the design notes)
    ref = _bf16_to_f32(d["x"][rows]).astype(np.float64) @ d["w"].astype(np.float64).T
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 0.1

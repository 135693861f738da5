"""GPU parity of the weight-only int4 (HQQ) path against the CPU oracle.

Packing and the standalone dequantization are bit-exact.  The fused GEMM
dequantizes inside the kernel and multiplies on the tensor cores (bf16 x bf16
-> fp32, kind::f16): each product is exact in fp32, the order of the fp32
sum is the hardware's, so the bf16 outputs are compared with the oracle's
exact (float64) sum within ACC_REL * sum_k |x_k w_k| plus one bf16 ulp.  A
one-hot activation makes the sum a single product, which must come back
bit-exact: that checks the dequantization inside the GEMM on its own.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_bits, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

dq = pytest.importorskip("quantized_gemm_token_b200") if torch.cuda.is_available() else None

# |acc - exact| <= ACC_REL * sum_k |x_k w_k|: 2^-20, sixteen times the fp32
# unit roundoff (a K-term sum rounded term by term can be off by up to
# (K-1) * 2^-24 of that sum; split partial sums add one rounding per split).
ACC_REL = 2.0 ** -20


@pytest.fixture(autouse=True)
def _sync_and_check():
    yield
    if torch.cuda.is_available():
        assert dq.dq_sync_status() == dq.DQ_OK


def _vals(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _ulp(v):
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def _assert_close(got_bits, exact, bound):
    got = _vals(got_bits)
    tol = _ulp(np.maximum(np.abs(exact), np.abs(got))) + ACC_REL * bound
    err = np.abs(got - exact)
    worst = np.max(err / tol) if err.size else 0.0
    assert worst <= 1.0, f"error {worst:.3f} of the bound at {np.unravel_index(np.argmax(err / tol), err.shape)}"


def _weights(d):
    packed = oracle.hqq_pack(d["codes"])
    w = oracle.hqq_dequant(packed, d["scale"], d["zero"], d["group"], signed=d["signed"])
    return packed, w


def _dev_weights(d, packed):
    """Packed codes and the group-major [K/group, N] scales and zero points."""
    return to_dev(packed), to_dev_bf16(d["scale"].T.copy()), to_dev_bf16(d["zero"].T.copy())


# ---------------------------------------------------------------- format

@pytest.mark.parametrize("R,C,signed", [(1, 2, False), (7, 40, True), (4096, 4096, False), (33, 4098, True)])
def test_pack_bit_exact(R, C, signed):
    lo, hi = (-8, 7) if signed else (0, 15)
    codes = synth.uniform_int8((R, C), lo, hi, 3 + C)
    p = dq.dq_hqq_pack(to_dev(codes))
    assert np.array_equal(p.cpu().numpy(), oracle.hqq_pack(codes))


@pytest.mark.parametrize("N,G", [(1, 1), (8, 2), (4096, 32), (136, 5), (33, 70)])
def test_group_major_bit_exact(N, G):
    m = synth.normal_bf16((N, G), 1.0, N + G)
    got = dq.dq_hqq_group_major(to_dev_bf16(m))
    assert np.array_equal(bf16_bits(got), m.T)


@pytest.mark.parametrize("N,K,group,signed", [(8, 64, 64, False), (24, 256, 32, True), (256, 4096, 128, False),
                                              (136, 1024, 256, True), (4096, 4096, 128, False)])
def test_dequantize_bit_exact(N, K, group, signed):
    d = synth.hqq(seed=N + K, M=1, N=N, K=K, group=group, signed=signed)
    packed, w = _weights(d)
    pk, sc, ze = _dev_weights(d, packed)
    got = dq.dq_hqq_dequantize(pk, sc, ze, group, signed=signed)
    assert np.array_equal(bf16_bits(got), w)


# ---------------------------------------------------------------- forward

FWD = [  # M, N, K, group, signed
    (1, 256, 256, 128, False),
    (16, 512, 1024, 128, False),      # few tiles: split contraction
    (33, 264, 320, 64, True),         # ragged channels, tokens and steps
    (200, 384, 512, 32, False),       # 208-token tiles
    (300, 128, 256, 256, True),       # two token tiles
    (257, 136, 96, 32, False),        # K = 96: half of the last step is padding
    (64, 1024, 2048, 128, True),      # eight splits (one cluster of 8 CTAs per tile)
    (40, 256, 2048, 64, False),       # eight splits of a 48-token tile: 6 tokens per CTA's reduction
    (1, 128, 4096, 32, True),         # one token, one tile, eight splits
]


@pytest.mark.parametrize("M,N,K,group,signed", FWD)
def test_linear_matches_oracle(M, N, K, group, signed):
    d = synth.hqq(seed=M + N, M=M, N=N, K=K, group=group, signed=signed)
    packed, w = _weights(d)
    pk, sc, ze = _dev_weights(d, packed)
    out = dq.dq_hqq_linear(to_dev_bf16(d["x"]), pk, sc, ze, group, signed=signed)
    exact = oracle.hqq_linear_f64(d["x"], w)
    bound = np.abs(_vals(d["x"])) @ np.abs(_vals(w)).T
    _assert_close(bf16_bits(out), exact, bound)


def test_linear_zero_tokens():
    d = synth.hqq(seed=1, M=1, N=64, K=128, group=64)
    packed, _ = _weights(d)
    pk, sc, ze = _dev_weights(d, packed)
    out = dq.dq_hqq_linear(torch.empty((0, 128), dtype=torch.bfloat16, device="cuda"), pk, sc, ze, 64)
    assert out.shape == (0, 64)


@pytest.mark.parametrize("signed", [False, True])
def test_one_hot_reads_dequantized_weight_exactly(signed):
    N, K, group = 264, 320, 64
    d = synth.hqq(seed=9, M=1, N=N, K=K, group=group, signed=signed)
    packed, w = _weights(d)
    pk, sc, ze = _dev_weights(d, packed)
    ks = np.arange(0, K, 3)
    x = np.zeros((len(ks), K), np.float32)
    x[np.arange(len(ks)), ks] = 1.0
    out = dq.dq_hqq_linear(to_dev_bf16(synth.f32_to_bf16_bits(x)), pk, sc, ze, group, signed=signed)
    assert np.array_equal(bf16_bits(out), w[:, ks].T)


@pytest.mark.parametrize("M", [16, 128, 1024])
def test_linear_full_size_every_token(M):
    """The benchmark shapes (N = K = 4096, group 128), oracle on every token."""
    N = K = 4096
    d = synth.hqq(seed=M, M=M, N=N, K=K, group=128)
    packed, w = _weights(d)
    pk, sc, ze = _dev_weights(d, packed)
    out = dq.dq_hqq_linear(to_dev_bf16(d["x"]), pk, sc, ze, 128)
    # every token (M <= 1024)
    exact = oracle.hqq_linear_f64(d["x"], w)
    bound = np.abs(_vals(d["x"])) @ np.abs(_vals(w)).T
    _assert_close(bf16_bits(out), exact, bound)


def test_split_contraction_is_deterministic():
    """The few-token split contraction (a cluster of CTAs per tile adding
    their partials in split order) gives identical bits on every call, and
    needs no workspace (a caller's buffer is accepted and ignored)."""
    M, N, K = 16, 4096, 4096
    assert dq.dq_hqq_workspace_size(M, N, K) == 0
    d = synth.hqq(seed=21, M=M, N=N, K=K, group=128)
    packed, _ = _weights(d)
    pk, sc, ze = _dev_weights(d, packed)
    x = to_dev_bf16(d["x"])
    junk = torch.full((1 << 20,), 0x5A, dtype=torch.uint8, device="cuda")
    a = bf16_bits(dq.dq_hqq_linear(x, pk, sc, ze, 128))
    b = bf16_bits(dq.dq_hqq_linear(x, pk, sc, ze, 128, workspace=junk))
    c = bf16_bits(dq.dq_hqq_linear(x, pk, sc, ze, 128))
    assert np.array_equal(a, b) and np.array_equal(a, c)
    assert int((junk != 0x5A).count_nonzero()) == 0


# ---------------------------------------------------------------- transposed

TRANS = [  # M, N, K, group, signed
    (16, 512, 1024, 128, False),
    (33, 264, 320, 64, True),
    (200, 384, 512, 32, False),
    (5, 72, 192, 64, False),          # contraction 72: a ragged step; 192 outputs: a ragged tile
    (24, 2048, 256, 64, True),        # eight splits of a 32-token tile
]


@pytest.mark.parametrize("M,N,K,group,signed", TRANS)
def test_linear_t_matches_oracle(M, N, K, group, signed):
    d = synth.hqq(seed=M + K, M=M, N=N, K=K, group=group, signed=signed)
    packed, w = _weights(d)
    pk, sc, ze = _dev_weights(d, packed)
    y = synth.normal_bf16((M, N), 1.0, 300 + M)
    out = dq.dq_hqq_linear_t(to_dev_bf16(y), pk, sc, ze, group, signed=signed)
    exact = oracle.hqq_linear_t_f64(y, w)
    bound = np.abs(_vals(y)) @ np.abs(_vals(w))
    _assert_close(bf16_bits(out), exact, bound)


@pytest.mark.parametrize("signed", [False, True])
def test_one_hot_t_reads_dequantized_weight_exactly(signed):
    N, K, group = 136, 384, 128
    d = synth.hqq(seed=10, M=1, N=N, K=K, group=group, signed=signed)
    packed, w = _weights(d)
    pk, sc, ze = _dev_weights(d, packed)
    ns = np.arange(N)
    y = np.zeros((N, N), np.float32)
    y[ns, ns] = 1.0
    out = dq.dq_hqq_linear_t(to_dev_bf16(synth.f32_to_bf16_bits(y)), pk, sc, ze, group, signed=signed)
    assert np.array_equal(bf16_bits(out), w)


def test_linear_t_full_size_every_token():
    M, N, K = 128, 4096, 4096
    d = synth.hqq(seed=77, M=1, N=N, K=K, group=128)
    packed, w = _weights(d)
    pk, sc, ze = _dev_weights(d, packed)
    y = synth.normal_bf16((M, N), 1.0, 78)
    out = dq.dq_hqq_linear_t(to_dev_bf16(y), pk, sc, ze, 128)
    # every token
    exact = oracle.hqq_linear_t_f64(y, w)
    bound = np.abs(_vals(y)) @ np.abs(_vals(w))
    _assert_close(bf16_bits(out), exact, bound)


# ---------------------------------------------------------------- layer and errors

def test_layer_forward_and_backward_input():
    M, N, K = 48, 256, 512
    d = synth.hqq(seed=5, M=M, N=N, K=K, group=64, signed=True)
    _, w = _weights(d)
    layer = dq.HqqLinear.from_codes(to_dev(d["codes"]), to_dev_bf16(d["scale"]), to_dev_bf16(d["zero"]), 64,
                                    signed=True)
    out = layer(to_dev_bf16(d["x"]))
    _assert_close(bf16_bits(out), oracle.hqq_linear_f64(d["x"], w),
                  np.abs(_vals(d["x"])) @ np.abs(_vals(w)).T)
    g = synth.normal_bf16((M, N), 1.0, 6)
    gi = layer.backward_input(to_dev_bf16(g))
    _assert_close(bf16_bits(gi), oracle.hqq_linear_t_f64(g, w), np.abs(_vals(g)) @ np.abs(_vals(w)))


def test_rejections_launch_nothing():
    lib = dq.lib
    pk = torch.zeros((64, 64), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((64, 2), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    P = lambda t: t.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    # group 48 does not exist; flags outside DQ_HQQ_S4; N not a multiple of 8
    assert lib.dq_hqq_linear(P(x), 4, P(pk), P(sc), P(sc), 64, 128, 48, 0, P(out), None, 0, s) == dq.DQ_ERR_INVALID_ARG
    assert lib.dq_hqq_linear(P(x), 4, P(pk), P(sc), P(sc), 64, 128, 64, 2, P(out), None, 0, s) == dq.DQ_ERR_INVALID_ARG
    assert lib.dq_hqq_linear(P(x), 4, P(pk), P(sc), P(sc), 60, 128, 64, 0, P(out), None, 0, s) == dq.DQ_ERR_UNSUPPORTED
    # misaligned activation pointer, K not a multiple of the group
    assert lib.dq_hqq_linear(P(x) + 2, 4, P(pk), P(sc), P(sc), 64, 128, 64, 0, P(out), None, 0, s) == dq.DQ_ERR_UNSUPPORTED
    assert lib.dq_hqq_linear(P(x), 4, P(pk), P(sc), P(sc), 64, 96, 64, 0, P(out), None, 0, s) == dq.DQ_ERR_INVALID_ARG
    assert lib.dq_hqq_pack(P(x), 3, 5, P(pk), s) == dq.DQ_ERR_INVALID_ARG

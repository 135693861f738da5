"""GPU parity of the 2:4 semi-structured sparse int8 path against the CPU
oracle: compression bit-exact (values, metadata, violation count), the int32
product bit-exact (int8 x int8 sums are exact and order-free), the bf16
epilogue within one bf16 ulp (the int8 layer's bar; measured identical)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import assert_bf16_close, bf16_bits, tile_rows, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

dq = pytest.importorskip("quantized_gemm_token_b200") if torch.cuda.is_available() else None


@pytest.fixture(autouse=True)
def _sync_and_check():
    yield
    if torch.cuda.is_available():
        assert dq.dq_sync_status() == dq.DQ_OK


def _random_s24(N, K, seed, sparse_groups=True):
    W = synth.uniform_int8((N, K), -127, 127, seed)
    W[~synth.s24_mask(N, K, seed + 3)] = 0
    if sparse_groups and N > 2 and K >= 16:
        W[1, :8] = 0                 # empty groups
        W[2, 4:8] = [0, 0, 9, 0]     # one nonzero
    return W


def _ws(M, N, K):
    n = dq.dq_s24_workspace_size(M, N, K)
    return torch.zeros((n,), dtype=torch.uint8, device="cuda") if n else None


@pytest.mark.parametrize("N,K", [(8, 8), (37, 256), (4096, 4096), (264, 1280)])
def test_compress_bit_exact(N, K):
    W = _random_s24(N, K, N + K)
    if N >= 37:
        W[5, 0:4] = [1, 2, 3, 0]     # a violation: three nonzeros
        W[6, 8:12] = [4, 5, 6, 7]    # four nonzeros
    viol = torch.zeros((1,), dtype=torch.int32, device="cuda")
    v, m = dq.dq_s24_compress(to_dev(W), violations=viol)
    vo, mo, bad = oracle.s24_compress(W)
    assert np.array_equal(v.cpu().numpy(), vo)
    assert np.array_equal(m.cpu().numpy(), mo)
    assert int(viol.item()) == bad


SHAPES = [(1, 256, 256), (16, 512, 1024), (33, 264, 384), (200, 384, 512), (300, 128, 256), (64, 1024, 2048),
          (513, 136, 128), (2, 8, 128)]


@pytest.mark.parametrize("use_ws", [True, False])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_linear_matches_oracle(M, N, K, use_ws):
    W = _random_s24(N, K, 7 + N)
    A = synth.uniform_int8((M, K), -127, 127, 8 + M)
    s_row = synth.uniform_f32((M,), 0.001, 0.05, 9)
    s_col = synth.uniform_f32((N,), 0.001, 0.05, 10)
    bias = synth.normal_bf16((N,), 0.1, 11)
    v, m, _ = oracle.s24_compress(W)
    vd, md, Ad = to_dev(v), to_dev(m), to_dev(A)
    ws = _ws(M, N, K) if use_ws else None
    acc = dq.dq_s24_int8_linear(Ad, None, vd, md, None, out_dtype="s32", workspace=ws)
    want = oracle.gemm_s32(A, oracle.s24_decompress(v, m))
    assert np.array_equal(acc.cpu().numpy(), want)
    for b in (None, bias):
        out = dq.dq_s24_int8_linear(Ad, to_dev(s_row), vd, md, to_dev(s_col),
                                    bias=None if b is None else to_dev_bf16(b), workspace=ws)
        assert_bf16_close(bf16_bits(out), oracle.epilogue_bf16(want, s_row, s_col, b))
    if ws is not None:
        # every completed call leaves the split arrival counters at zero: one
        # more call with the same workspace writes every output element (a
        # counter left behind would keep the last split from storing)
        out = torch.full((M, N), 0x7FFFFFFF, dtype=torch.int32, device="cuda")
        dq.dq_s24_int8_linear(Ad, None, vd, md, None, out=out, out_dtype="s32", workspace=ws)
        assert np.array_equal(out.cpu().numpy(), want)


@pytest.mark.parametrize("M,N,K", [(300, 264, 256), (513, 1032, 1024), (1600, 4104, 2048), (40, 512, 384)])
def test_pair_kernel_matches_oracle(M, N, K):
    """The 2-SM pair kernel (tcgen05.mma.sp over two SMs, each CTA's
    metadata copied into its own tensor memory), forced with schedule 3 and
    automatic from 1536 tokens and K >= 2048: int32 bit-exact and the bf16
    epilogue with bias, on ragged channels (a pair tile whose second half
    lies past N), tokens and both token-tile halves."""
    W = _random_s24(N, K, 17 + N)
    A = synth.uniform_int8((M, K), -127, 127, 18 + M)
    s_row = synth.uniform_f32((M,), 0.001, 0.05, 19)
    s_col = synth.uniform_f32((N,), 0.001, 0.05, 20)
    bias = synth.normal_bf16((N,), 0.1, 21)
    v, m, _ = oracle.s24_compress(W)
    vd, md, Ad = to_dev(v), to_dev(m), to_dev(A)
    want = oracle.gemm_s32(A, oracle.s24_decompress(v, m))
    dq.dq_debug_set_schedule(3)
    try:
        acc = dq.dq_s24_int8_linear(Ad, None, vd, md, None, out_dtype="s32")
        out = dq.dq_s24_int8_linear(Ad, to_dev(s_row), vd, md, to_dev(s_col), bias=to_dev_bf16(bias))
    finally:
        dq.dq_debug_set_schedule(0)
    assert np.array_equal(acc.cpu().numpy(), want)
    assert_bf16_close(bf16_bits(out), oracle.epilogue_bf16(want, s_row, s_col, bias))


@pytest.mark.parametrize("M,K,N", [(2048, 4096, 4096), (16, 8192, 28672)])
def test_layer_full_size(M, K, N):
    """The benchmark shapes: quantize (GPU), compress (GPU), sparse product;
    the oracle on every token (M = 16) or on 1024 tokens covering both edges
    of every 128-row tile (M = 2048)."""
    d = synth.s24(0, M=M, K=K, N=N)
    x = to_dev_bf16(d["x"])
    q, s = dq.dq_quantize_rows(x)
    wq, sc = dq.dq_quantize_weight(to_dev(d["w"]))
    v, m = dq.dq_s24_compress(wq)
    out = dq.dq_s24_int8_linear(q, s, v, m, sc, workspace=_ws(M, N, K))
    qo, so = oracle.quantize_rows_bf16(d["x"])
    wo, sco = oracle.quantize_rows_f32(d["w"])
    assert np.array_equal(wq.cpu().numpy(), wo)
    assert np.array_equal(q.cpu().numpy(), qo)
    rows = tile_rows(M)                         # every token for M = 16; 1024 rows (all M-tile edges) for 2048
    want = oracle.linear_bf16(qo[rows], so[rows], wo, sco)
    assert_bf16_close(bf16_bits(out)[rows], want)


def test_rejections_launch_nothing():
    lib = dq.lib
    A = torch.zeros((4, 256), dtype=torch.int8, device="cuda")
    v = torch.zeros((64, 128), dtype=torch.int8, device="cuda")
    m = torch.zeros((64, 32), dtype=torch.uint8, device="cuda")
    out = torch.zeros((4, 64), dtype=torch.int32, device="cuda")
    P = lambda t: t.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    # K not a multiple of 128; N not a multiple of 8; unknown output type
    assert lib.dq_s24_int8_linear(P(A), None, 4, 192, P(v), P(m), None, 64, None, P(out), 1, None, 0, s) == dq.DQ_ERR_UNSUPPORTED
    assert lib.dq_s24_int8_linear(P(A), None, 4, 256, P(v), P(m), None, 60, None, P(out), 1, None, 0, s) == dq.DQ_ERR_UNSUPPORTED
    assert lib.dq_s24_int8_linear(P(A), None, 4, 256, P(v), P(m), None, 64, None, P(out), 7, None, 0, s) == dq.DQ_ERR_INVALID_ARG
    assert lib.dq_s24_compress(P(A), 4, 12, P(v), P(m), None, s) == dq.DQ_ERR_INVALID_ARG


def test_layer_class_matches_oracle():
    """S24Int8Linear: weight quantized and compressed once, tokens quantized per call."""
    N, K = 256, 1024
    d = synth.s24(1, M=48, K=K, N=N)
    bias = synth.normal_bf16((N,), 0.1, 12)
    layer = dq.S24Int8Linear.from_float(to_dev(d["w"]), bias=to_dev_bf16(bias))
    wo, sco = oracle.quantize_rows_f32(d["w"])
    for M in (48, 16):                      # 16 tokens split the contraction
        x = d["x"][:M]
        out = layer(to_dev_bf16(x))
        qo, so = oracle.quantize_rows_bf16(x)
        assert_bf16_close(bf16_bits(out), oracle.linear_bf16(qo, so, wo, sco, bias))

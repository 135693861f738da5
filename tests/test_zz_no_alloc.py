"""The allocation-free entry point dq_int8_linear_noalloc, called through the
C ABI, against dq_int8_linear with a caller-owned workspace.

It exists for callers that cannot allocate device memory (an engine whose
memory planner owns all device memory, code running during another
component's CUDA-graph capture, latency-bound callers that cannot afford the
synchronisation of cudaMalloc/cudaFree): its split-K scratch is a static
32 MiB device array inside libdq.  This file is collected last on purpose;
it needs nothing from the other tests and passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, seed):
    A = synth.uniform_int8((M, K), -127, 127, seed)
    W = synth.uniform_int8((N, K), -127, 127, seed + 1)
    s_row = synth.uniform_f32((M,), 0.001, 0.05, seed + 5)
    s_col = synth.uniform_f32((N,), 0.001, 0.05, seed + 6)
    bias = synth.normal_bf16((N,), 0.1, seed + 2)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    b = torch.from_numpy(bias.view(np.int16)).view(torch.bfloat16).cuda()
    return dev(A), dev(W), dev(s_row), dev(s_col), b


def _call_noalloc(lib, A, s_row, W, s_col, bias, out, code):
    M, K = A.shape
    N = W.shape[0]
    P = ctypes.c_void_p
    ptr = lambda t: None if t is None else P(t.data_ptr())  # noqa: E731
    stream = P(torch.cuda.current_stream().cuda_stream)
    return lib.dq_int8_linear_noalloc(ptr(A), ptr(s_row), ctypes.c_int64(M), ctypes.c_int64(K), ptr(W),
                                      ptr(s_col), ctypes.c_int64(N), ptr(bias), ptr(out), ctypes.c_int(code),
                                      stream)


# (M, N, K, uses the scratch): few-token shapes whose (swap-AB) stream-K
# schedule uses 0.5 MB and 8.4 MB of scratch, and one whose schedule needs
# none (the call goes straight to the plain entry point)
@pytest.mark.parametrize("M,N,K,uses", [(16, 8192, 8192, True), (128, 16384, 8192, True), (256, 256, 256, False)])
def test_noalloc_matches_workspace_entry_two_calls(M, N, K, uses):
    import quantized_gemm_token_b200 as dq
    from gpu_util import assert_bf16_close, bf16_bits
    lib = dq.lib
    need = dq.dq_int8_linear_workspace_size(M, N, K)
    assert need <= dq.DQ_NOALLOC_SCRATCH_BYTES
    assert (need > 0) == uses
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    for call, seed in enumerate((900, 950)):             # two calls in a row, different data
        A, W, s_row, s_col, bias = _inputs(M, N, K, seed)
        ref32 = dq.dq_int8_linear(A, None, W, None, out_dtype="s32", workspace=ws)
        ref16 = dq.dq_int8_linear(A, s_row, W, s_col, bias=bias, workspace=ws)
        out32 = torch.empty((M, N), dtype=torch.int32, device="cuda")
        out16 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(lib, A, None, W, None, None, out32, dq.DQ_OUT_S32) == dq.DQ_OK
        assert _call_noalloc(lib, A, s_row, W, s_col, bias, out16, dq.DQ_OUT_BF16) == dq.DQ_OK
        assert dq.dq_sync_status() == dq.DQ_OK
        assert torch.equal(out32, ref32), f"call {call}: int32 differs"
        assert_bf16_close(bf16_bits(out16), bf16_bits(ref16))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """With the automatic plan no shape needs more scratch than the entry
    point has (wide few-token shapes take the dense arrangement, which needs
    none); forcing the swap-AB stream-K schedule on a wide one does, and the
    call must then refuse rather than overrun the array."""
    import quantized_gemm_token_b200 as dq
    M, N, K = 128, 66560, 256
    assert dq.dq_int8_linear_workspace_size(M, N, K) == 0
    dq.dq_debug_set_schedule(2)                           # swap-AB, stream-K: ~34 MB of scratch
    try:
        assert dq.dq_int8_linear_workspace_size(M, N, K) > dq.DQ_NOALLOC_SCRATCH_BYTES
        A, W, s_row, s_col, bias = _inputs(M, N, K, 990)
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(dq.lib, A, s_row, W, s_col, None, out, dq.DQ_OUT_BF16) == dq.DQ_ERR_UNSUPPORTED
    finally:
        dq.dq_debug_set_schedule(0)


def test_noalloc_rejects_what_the_plain_entry_rejects():
    """Arguments the plain entry point refuses (K not a multiple of 16, a bad
    output type, negative M) get the same status, before any launch."""
    import quantized_gemm_token_b200 as dq
    lib = dq.lib
    P = ctypes.c_void_p
    M, N, K = 16, 8192, 8200                      # K % 16 != 0
    A, W, s_row, s_col, _ = _inputs(M, N, 8192, 991)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    stream = P(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: P(t.data_ptr())  # noqa: E731
    for (m, k, code) in ((M, K, dq.DQ_OUT_BF16), (M, 8192, 7), (-1, 8192, dq.DQ_OUT_BF16)):
        args = (ptr(A), ptr(s_row), ctypes.c_int64(m), ctypes.c_int64(k), ptr(W), ptr(s_col), ctypes.c_int64(N),
                None, ptr(out), ctypes.c_int(code))
        plain = lib.dq_int8_linear(*args, None, ctypes.c_size_t(0), stream)
        assert plain != dq.DQ_OK
        assert lib.dq_int8_linear_noalloc(*args, stream) == plain
    assert dq.dq_sync_status() == dq.DQ_OK


def test_noalloc_python_wrapper_checks_and_matches():
    """The binding's dq_int8_linear_noalloc checks its tensors like
    dq_int8_linear (a wrong output type or shape raises, nothing launches)
    and returns the same result, twice in a row."""
    import quantized_gemm_token_b200 as dq
    from gpu_util import assert_bf16_close, bf16_bits
    M, N, K = 16, 8192, 8192
    A, W, s_row, s_col, bias = _inputs(M, N, K, 993)
    with pytest.raises(TypeError):
        dq.dq_int8_linear_noalloc(A, s_row, W, s_col, torch.empty((M, N), dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError):
        dq.dq_int8_linear_noalloc(A, s_row, W, s_col, torch.empty((M, N - 8), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        dq.dq_int8_linear_noalloc(A, s_row, W[:, :K - 16].contiguous(), s_col,
                                  torch.empty((M, N), dtype=torch.bfloat16, device="cuda"))
    ws = torch.zeros(dq.dq_int8_linear_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
    ref = dq.dq_int8_linear(A, s_row, W, s_col, bias=bias, workspace=ws)
    for _ in range(2):
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        dq.dq_int8_linear_noalloc(A, s_row, W, s_col, out, bias=bias)
        assert_bf16_close(bf16_bits(out), bf16_bits(ref))
    assert dq.dq_sync_status() == dq.DQ_OK

"""The tcgen05 projection GEMM (prefill) against a float64 NumPy matmul of the
same BF16 operands, through the C ABI, on shapes with ragged M and N tails
and on the Dory projection shapes."""
import ctypes

import numpy as np
import pytest
import torch

from looped_ngpt_b200 import _lib
from synthetic.gen import f32_to_bf16_bits, bf16_bits_to_f32

pytestmark = pytest.mark.gpu


def _bf16(rng, shape, scale=1.0):
    return f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * scale)


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (64, 640, 256), (200, 300, 128),
                                   (129, 257, 192), (512, 6400, 2560),
                                   (256, 2560, 10240)])
def test_gemm_matches_numpy(M, N, K):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    A = _bf16(rng, (M, K))
    W = _bf16(rng, (N, K), 1.0 / np.sqrt(K))
    dA = torch.from_numpy(A.view(np.int16)).cuda()
    dW = torch.from_numpy(W.view(np.int16)).cuda()
    dC = torch.full((M, N), float("nan"), device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    lib = _lib.load()
    assert lib.dory_debug_gemm_bf16(ctypes.c_void_p(dA.data_ptr()), K,
                                    ctypes.c_void_p(dW.data_ptr()),
                                    ctypes.c_void_p(dC.data_ptr()), M, N, K, s) == 0
    torch.cuda.synchronize()
    ref = bf16_bits_to_f32(A).astype(np.float64) @ bf16_bits_to_f32(W).astype(np.float64).T
    got = dC.cpu().numpy()
    # f32 accumulation of K products of magnitude ~|ref|/sqrt(K)
    tol = 1e-5 * np.sqrt(K) * (np.abs(ref).max() + 1)
    assert np.abs(got - ref).max() <= tol, np.abs(got - ref).max()


@pytest.mark.parametrize("M,N,K", [(64, 2560, 10240), (64, 2560, 2560),
                                   (64, 6400, 2560), (10, 640, 256),
                                   (1, 300, 192)])
def test_gemm_k_split_partials_sum_to_product(M, N, K):
    """Decode-batch shapes (one row tile, few column tiles): K is split
    across SMs and the partial slabs must sum to the product; the split
    count follows the tile count (about one work item per SM)."""
    rng = np.random.default_rng(M * 11 + N * 5 + K)
    A = _bf16(rng, (M, K))
    W = _bf16(rng, (N, K), 1.0 / np.sqrt(K))
    dA = torch.from_numpy(A.view(np.int16)).cuda()
    dW = torch.from_numpy(W.view(np.int16)).cuda()
    S = 16
    dC = torch.full((S, M, N), float("nan"), device="cuda")
    n = ctypes.c_int(0)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    lib = _lib.load()
    assert lib.dory_debug_gemm_bf16_split(
        ctypes.c_void_p(dA.data_ptr()), K, ctypes.c_void_p(dW.data_ptr()),
        ctypes.c_void_p(dC.data_ptr()), M, N, K, S, ctypes.byref(n), s) == 0
    torch.cuda.synchronize()
    tiles = -(-N // 256)
    kb = K // 64
    assert 1 <= n.value <= min(S, kb)
    if tiles * 2 <= torch.cuda.get_device_properties(0).multi_processor_count and kb >= 4:
        assert n.value > 1, "a decode-batch shape must be split"
    got = dC[: n.value].sum(0).cpu().numpy().astype(np.float64)
    assert not np.isnan(dC[: n.value].cpu().numpy()).any()
    ref = bf16_bits_to_f32(A).astype(np.float64) @ bf16_bits_to_f32(W).astype(np.float64).T
    tol = 1e-5 * np.sqrt(K) * (np.abs(ref).max() + 1)
    assert np.abs(got - ref).max() <= tol, np.abs(got - ref).max()


def test_gemm_misaligned_operand_reports_error():
    """A operand 2 bytes past a 16-byte boundary: the TMA descriptor cannot be
    built, nothing is launched, the call returns DORY_ERR_CUDA and the
    output keeps its contents."""
    M, N, K = 64, 256, 128
    buf = torch.zeros(M * K + 8, dtype=torch.int16, device="cuda")
    dW = torch.zeros((N, K), dtype=torch.int16, device="cuda")
    dC = torch.full((M, N), float("nan"), device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    lib = _lib.load()
    assert lib.dory_debug_gemm_bf16(ctypes.c_void_p(buf.data_ptr() + 2), K,
                                    ctypes.c_void_p(dW.data_ptr()),
                                    ctypes.c_void_p(dC.data_ptr()), M, N, K,
                                    s) == -4
    torch.cuda.synchronize()
    assert torch.isnan(dC).all()

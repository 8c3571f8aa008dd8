"""The tcgen05 GEMM kernel through its test hook: every operand-major
combination, both tile widths and both operand types (bf16, fp16) against an
fp64 product of the same operands (plus fp32-accumulation rounding)."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import folded_tensor_sequence_map_b200 as T


def _bf16(shape, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(dtype)


@pytest.mark.parametrize("f16", [False, True])
@pytest.mark.parametrize("a_mn,b_mn", [(False, False), (False, True), (True, True), (True, False)])
@pytest.mark.parametrize("M,N,K,bn128", [(128, 128, 64, False), (256, 256, 192, False), (384, 512, 1024, False),
                                         (256, 384, 320, True), (1024, 768, 512, True)])
def test_gemm_matches_fp64(a_mn, b_mn, M, N, K, bn128, f16):
    dt = torch.float16 if f16 else torch.bfloat16
    A = _bf16((K, M) if a_mn else (M, K), 1, dt)
    B = _bf16((K, N) if b_mn else (N, K), 2, dt)
    Am = A.double().T if a_mn else A.double()
    Bm = B.double() if b_mn else B.double().T
    ref = (Am @ Bm).numpy()
    C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    T.tsp_test_gemm(a_mn, b_mn, M, N, K, A.cuda(), A.shape[1], B.cuda(), B.shape[1], C, N, bn128, f16=f16)
    torch.cuda.synchronize()
    got = C.cpu().double().numpy()
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert np.isfinite(got).all() and err < 1e-5, err


def test_gemm_many_tiles_persistent():
    # more tiles than SMs: the persistent scheduler and both TMEM buffers are exercised
    M, N, K = 4096, 2048, 256
    A, B = _bf16((M, K), 3), _bf16((N, K), 4)
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    T.tsp_test_gemm(False, False, M, N, K, A.cuda(), K, B.cuda(), K, C, N)
    ref = (A.cuda().float() @ B.cuda().float().T)
    err = ((C - ref).abs().max() / ref.abs().max()).item()
    assert err < 1e-5, err

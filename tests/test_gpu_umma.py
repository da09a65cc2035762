"""Tensor-core building blocks (tcgen05 MMA from the library's shared-memory
layouts, TMEM accumulators) checked through lola_selftest_umma against a
float64 matrix product."""
import ctypes

import pytest
import torch

import sparse_kv_caching_b200 as lola

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _run(mode, N, K, seed=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    tf32 = bool(mode & 2)
    A = torch.randn(128, K, generator=g)
    B = torch.randn(K, N, generator=g)
    if not tf32:
        A, B = A.bfloat16(), B.bfloat16()
    Bin = B if mode & 1 else B.t().contiguous()
    Ad, Bd = A.cuda(), Bin.cuda()
    C = torch.full((128, N), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L = lola.lib()
    rc = L.lola_selftest_umma(mode, ctypes.c_void_p(Ad.data_ptr()), ctypes.c_void_p(Bd.data_ptr()),
                              ctypes.c_void_p(C.data_ptr()), 128, N, K, ctypes.c_void_p(err.data_ptr()),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, L.lola_last_error_string().decode()
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = A.double() @ B.double()
    return C.double().cpu(), ref


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("N,K", [(128, 128), (64, 64), (256, 32), (16, 16), (128, 256)])
def test_bf16(mode, N, K):
    C, ref = _run(mode, N, K)
    assert torch.isfinite(C).all()
    assert (C - ref).abs().max() / ref.abs().max() < 1e-5


# tf32 operands are used K-major only (the MN-major tf32 form is not used by
# the library and is not tested).
@pytest.mark.parametrize("mode", [2])
@pytest.mark.parametrize("N,K", [(128, 128), (64, 8), (32, 64)])
def test_tf32(mode, N, K):
    C, ref = _run(mode, N, K)
    assert (C - ref).abs().max() / ref.abs().max() < 5e-3


@pytest.mark.parametrize("mode", [6])
@pytest.mark.parametrize("N,K", [(128, 64), (64, 128), (16, 8), (128, 32)])
def test_3xtf32(mode, N, K):
    C, ref = _run(mode, N, K)
    assert (C - ref).abs().max() / ref.abs().max() < 1e-5

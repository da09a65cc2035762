"""Tensor-core building blocks (tcgen05 MMA from the library's shared-memory
layouts, TMEM accumulators) checked through lola_selftest_umma against a
float64 matrix product, and the bounded-wait failure path: a completion wait
that nothing will satisfy gives up, the kernel returns, and the state's sync
point reports LOLA_ERR_TIMEOUT."""
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


def _run(mode, N, K, seed=0, err=None):
    g = torch.Generator(device="cpu").manual_seed(seed)
    tf32 = bool(mode & 2)
    A = torch.randn(128, K, generator=g)
    B = torch.randn(K, N, generator=g)
    if not tf32:
        A, B = A.bfloat16(), B.bfloat16()
    Bin = B if mode & 1 else B.t().contiguous()
    Ain = A.t().contiguous() if mode & 8 else A
    Ad, Bd = Ain.cuda(), Bin.cuda()
    C = torch.full((128, N), float("nan"), device="cuda")
    if err is None:
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L = lola.lib()
    rc = L.lola_selftest_umma(mode, ctypes.c_void_p(Ad.data_ptr()), ctypes.c_void_p(Bd.data_ptr()),
                              ctypes.c_void_p(C.data_ptr()), 128, N, K, ctypes.c_void_p(err.data_ptr()),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, L.lola_last_error_string().decode()
    torch.cuda.synchronize()
    if mode & 32:
        return C, err
    assert err.item() == 0
    ref = A.double() @ B.double()
    return C.double().cpu(), ref


# modes 8, 9: A given MN-major ([K][M]), the layout of the fold's value operand
@pytest.mark.parametrize("mode", [0, 1, 8, 9])
@pytest.mark.parametrize("N,K", [(128, 128), (64, 64), (256, 32), (16, 16), (128, 256)])
def test_bf16(mode, N, K):
    C, ref = _run(mode, N, K)
    assert torch.isfinite(C).all()
    assert (C - ref).abs().max() / ref.abs().max() < 1e-5


# modes 64 + (0, 1, 8, 9): the 128-byte swizzled layout, in which the output
# kernel holds its key tiles (K-major for Q K^T, MN-major for P V)
@pytest.mark.parametrize("mode", [64, 65, 72, 73])
@pytest.mark.parametrize("N,K", [(128, 128), (64, 64), (256, 64), (128, 256)])
def test_bf16_swizzled(mode, N, K):
    C, ref = _run(mode, N, K)
    assert torch.isfinite(C).all()
    assert (C - ref).abs().max() / ref.abs().max() < 1e-5


# bf16 with A in tensor memory (two elements per column), the form of the
# output kernel's P V product (A = P; B = V MN-major, chunk-major or swizzled)
@pytest.mark.parametrize("mode", [16, 17, 80, 81])
@pytest.mark.parametrize("N,K", [(128, 64), (64, 128), (256, 64), (128, 128)])
def test_bf16_a_in_tmem(mode, N, K):
    C, ref = _run(mode, N, K)
    assert torch.isfinite(C).all()
    assert (C - ref).abs().max() / ref.abs().max() < 1e-5


# tf32 in the swizzled layout, K-major: plain, 3xTF32, and with A in tensor
# memory (the chain's SRE form: A = H^T parts in tensor memory, B = phi rows)
@pytest.mark.parametrize("mode", [66, 70, 82, 86])
@pytest.mark.parametrize("N,K", [(64, 128), (128, 64), (64, 32), (256, 64)])
def test_tf32_swizzled(mode, N, K):
    C, ref = _run(mode, N, K)
    tol = 1e-5 if mode & 4 else 5e-3
    assert torch.isfinite(C).all()
    assert (C - ref).abs().max() / ref.abs().max() < tol


# kind::tf32 reads the top 19 bits of an f32 operand: 3xTF32 with the hi parts
# passed raw equals 3xTF32 with them rounded down first, bit for bit (the
# chain's SRE hands its raw phi tile to the tensor cores as the hi part)
@pytest.mark.parametrize("mode", [6, 22, 70, 86])
@pytest.mark.parametrize("N,K", [(64, 128), (128, 64)])
def test_tf32_reads_the_top_19_bits(mode, N, K):
    C0, _ = _run(mode, N, K, seed=3)
    C1, _ = _run(mode | 128, N, K, seed=3)
    assert torch.equal(C0, C1)


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


# A read from tensor memory (row m in lane m), B from shared memory: the SRE
# product of the memory-update chain keeps H^T resident in tensor memory.
@pytest.mark.parametrize("mode", [18, 22])
@pytest.mark.parametrize("N,K", [(64, 128), (128, 64), (16, 16), (256, 64)])
def test_tf32_a_in_tmem(mode, N, K):
    C, ref = _run(mode, N, K)
    tol = 1e-5 if mode & 4 else 5e-3
    assert (C - ref).abs().max() / ref.abs().max() < tol


def test_bounded_wait_gives_up_and_reports():
    C, err = _run(2 | 32, 64, 64)
    assert err.item() == 1
    assert torch.isnan(C).all()


def test_timeout_surfaces_through_the_state_sync_point():
    """The state's error word set by a kernel whose bounded wait gave up makes
    lola_state_check (the sync point) return LOLA_ERR_TIMEOUT; a reset clears it."""
    import synth
    from tests import parity as P
    w = P.small_workload(2, B=1, Hkv=1, Hq=2, T=128, eta=64, lam=32, chunk=64)
    dev = P.to_device(w, synth.full_arrays(w))
    layer = P.make_layer(w, dev["W"])
    layer.prefill(dev["q"][:, :w.T].contiguous(), dev["k"][:, :w.T].contiguous(), dev["v"][:, :w.T].contiguous())
    layer.check()                                  # a healthy call reports nothing
    word = layer.export()["err_word"]
    _run(2 | 32, 64, 64, err=word)                 # a wait that gives up, writing the state's word
    with pytest.raises(lola.LolaError, match="TIMEOUT"):
        layer.check()
    layer.reset()
    layer.check()
    layer.close()

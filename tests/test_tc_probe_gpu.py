"""The tcgen05 wrappers (descriptors, TMEM layout, MMA, commit, TMEM loads)
checked through a test-only one-tile probe against a plain matrix product."""
import ctypes
import os

import pytest
import torch

pytestmark = pytest.mark.gpu


def _load_builder():
    """The probe's build module, loaded by path under its own name (both
    probe directories have a build.py)."""
    import importlib.util
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tc_probe", "build.py")
    spec = importlib.util.spec_from_file_location("tc_probe_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod



@pytest.fixture(scope="module")
def probe():
    probe_build = _load_builder()
    lib = ctypes.CDLL(probe_build.build())
    lib.tc_gemm_probe.restype = ctypes.c_int
    lib.tc_gemm_probe.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5 + [ctypes.c_void_p] * 2
    return lib


@pytest.mark.parametrize("M,N,K", [(128, 64, 128), (128, 128, 64), (128, 256, 128), (128, 192, 64), (128, 16, 16),
                                   (64, 64, 128), (64, 128, 64)])
@pytest.mark.parametrize("negate,twice", [(0, 0), (1, 1)], ids=["plain", "neg_acc"])
def test_tile_product_matches_matmul(probe, M, N, K, negate, twice):
    g = torch.Generator().manual_seed(M * 1000 + N * 10 + K)
    A = torch.randn(M, K, generator=g).bfloat16().cuda()
    B = torch.randn(N, K, generator=g).bfloat16().cuda()
    D = torch.full((M, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = probe.tc_gemm_probe(A.data_ptr(), B.data_ptr(), D.data_ptr(), M, N, K, negate, twice, status.data_ptr(),
                             torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0 and int(status.item()) == 0
    ref = (A.double() @ B.double().T) * (-1.0 if negate else 1.0) * (2.0 if twice else 1.0)
    err = (D.double() - ref).abs().max().item()
    assert err <= 1e-4 * max(1.0, ref.abs().max().item()), err


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (128, 64, 64), (64, 128, 128)])
@pytest.mark.parametrize("a_mn,b_mn", [(1, 0), (0, 1), (1, 1)], ids=["A_mn", "B_mn", "AB_mn"])
def test_mn_major_operands(probe, M, N, K, a_mn, b_mn):
    """Operands stored MN-major (16-byte rows of 8 consecutive M or N elements
    at one K index) with the descriptor's leading byte offset set to the
    stride between core matrices along K and the stride byte offset to the
    stride along M / N -- the same rule as for K-major operands."""
    probe.tc_gemm_probe_mn.restype = ctypes.c_int
    probe.tc_gemm_probe_mn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 6 + [ctypes.c_void_p] * 2
    g = torch.Generator().manual_seed(M + N + K + 7 * a_mn + 3 * b_mn)
    A = torch.randn(M, K, generator=g).bfloat16().cuda()
    B = torch.randn(N, K, generator=g).bfloat16().cuda()
    D = torch.full((M, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = probe.tc_gemm_probe_mn(A.data_ptr(), B.data_ptr(), D.data_ptr(), M, N, K, a_mn, b_mn, 1,
                                status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0 and int(status.item()) == 0
    ref = A.double() @ B.double().T
    err = (D.double() - ref).abs().max().item()
    assert err <= 1e-4 * max(1.0, ref.abs().max().item()), err

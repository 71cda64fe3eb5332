"""tcgen05 operand views used by the tensor-core forward kernel, checked with a
single-CTA GEMM (tests/csrc/tc_selftest.cu) against a float64 product of the
same fp16-rounded operands."""
import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "tc_selftest.cu")
LIB = os.path.join(HERE, "csrc", "libtc_selftest.so")


def build_selftest():
    hdr = os.path.join(ROOT, "channel_gated_delta_b200", "csrc", "tc_common.cuh")
    if os.path.exists(LIB) and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC), os.path.getmtime(hdr)):
        return LIB
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2",
                           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I",
                           os.path.join(ROOT, "channel_gated_delta_b200", "csrc"), "-I",
                           os.path.join(ROOT, "include"), SRC, "-o", LIB])
    return LIB


@pytest.fixture(scope="module")
def lib():
    l = ctypes.CDLL(build_selftest())
    l.tc_selftest.restype = ctypes.c_int
    l.tc_selftest.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 11 + [ctypes.c_void_p] * 2
    return l


# (M, N, K, a_mn, b_mn, a_neg, RA, a_row0, RB, b_row0, what[, d_lane])
CASES = [
    (128, 128, 128, 0, 0, 0, 128, 0, 128, 0, "decay products: K-major A and B"),
    (64, 128, 64, 0, 1, 0, 64, 0, 128, 0, "W' = Tinv Kp: MN-major B from the top half of a 128-row tile"),
    (64, 64, 64, 0, 1, 0, 64, 0, 64, 0, "N = Tinv M"),
    (128, 64, 64, 1, 1, 1, 128, 64, 64, 0, "-Khat^T R: MN-major A from rows 64..127, negated"),
    (128, 64, 64, 1, 1, 0, 128, 0, 64, 0, "K^T V: MN-major A and B"),
    (128, 64, 64, 0, 1, 1, 192, 64, 64, 0, "-[Aq;Bq] R: K-major A from rows 64..191 of a 192-row tile"),
    (128, 128, 128, 0, 1, 0, 128, 0, 128, 0, "[W';Q] S_c: MN-major B with two column blocks"),
    (128, 64, 128, 0, 1, 0, 128, 0, 128, 0, "[W';Q] S_c, one value half"),
    (128, 256, 64, 0, 0, 0, 128, 0, 256, 0, "N = 256, K-major B"),
    (64, 192, 64, 0, 1, 0, 64, 0, 64, 0, "N = 192, MN-major B with three column blocks"),
    (64, 64, 64, 0, 1, 0, 64, 0, 64, 0, "M = 64 accumulator in the upper half of each lane quadrant", 16),
]


@pytest.mark.parametrize("case", CASES, ids=[c[10] for c in CASES])
def test_tcgen05_operand_view(lib, case):
    M, N, K, a_mn, b_mn, a_neg, RA, a_row0, RB, b_row0 = case[:10]
    d_lane = case[11] if len(case) > 11 else 0
    g = torch.Generator().manual_seed(M * 7 + N + K + a_row0)
    A = torch.randn(M, K, generator=g)
    B = torch.randn(K, N, generator=g)
    ref = (A.half().double() @ B.half().double()) * (-1.0 if a_neg else 1.0)
    dA, dB = A.cuda(), B.cuda()
    dD = torch.full((M, N), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.tc_selftest(dA.data_ptr(), dB.data_ptr(), dD.data_ptr(), M, N, K, a_mn, b_mn, a_neg, RA, a_row0,
                         RB, b_row0, d_lane, err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0, "mbarrier wait ran out"
    D = dD.cpu().double()
    assert torch.isfinite(D).all()
    rel = (D - ref).abs().max() / ref.abs().max()
    assert rel < 1e-5, float(rel)

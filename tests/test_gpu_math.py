"""Direct checks of the verify kernels' hand-written fast-math helpers.

The kernels compute most softmax exponentials with the special-function
unit's 2^x, one pair in eight with a polynomial on the FMA pipe, and the
exponential variates of their Gumbel-max draws with a short series near
u' = 1.  The probes in csrc/sv_math_probe.cu run those helpers from the
library's own device header over dense grids; the results are compared with
fp64 here.  Bounds (relative error):
  ex2_poly_x2     2.5e-7 on [-126, 0]: the degree-5 Chebyshev interpolant's
                  own error is at most (ln 2)^6 sqrt(2) / (6! 2^5 2^6) = 1.1e-7
                  absolute on [-1/2, 1/2] (1.5e-7 relative), plus a few fp32
                  roundings of the Horner steps
  ex2f            2 ulp (2.4e-7) on [-126, 0]
  neg_exp1_log2   2 ulp (2.4e-7) where the series is used (v = 1 - u' < 1/8:
                  the degree-4 interpolant's own error is 1.4e-8, the four
                  fp32 Horner steps and the final product add the rest), 1e-6
                  where the hardware lg2 is (there |lg2 u'| >= 0.19 and lg2's
                  absolute error is about 2^-22.6); the two-at-a-time form
                  gives the same bits
A relative error of 2.4e-7 in an exponential variate moves a Gumbel-max
score by about 3.5e-7 (log2 units), far below the 1e-5 near-tie margin.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "csrc", "sv_math_probe.cu")
BUILD = os.path.join(ROOT, "tests", "_build")
LIB = os.path.join(BUILD, "libsvmathprobe.so")
DEVICE_HEADERS = [os.path.join(ROOT, "speculative_decoding_verification_88_b200", "csrc", h)
                  for h in ("sv_device.cuh", "sv_internal.h")]

pytestmark = pytest.mark.gpu


def build_probe() -> str:
    from speculative_decoding_verification_88_b200 import build as libbuild

    deps = [SRC] + DEVICE_HEADERS
    if os.path.exists(LIB) and all(os.path.getmtime(d) <= os.path.getmtime(LIB) for d in deps):
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([libbuild.nvcc_path(), *libbuild.NVCC_FLAGS,
                    "-I" + os.path.join(ROOT, "speculative_decoding_verification_88_b200", "csrc"),
                    "-I" + os.path.join(ROOT, "include"), "-o", tmp, SRC], check=True)
    os.replace(tmp, LIB)
    return LIB


@pytest.fixture(scope="module")
def probe():
    lib = ctypes.CDLL(build_probe())
    P, I64 = ctypes.c_void_p, ctypes.c_longlong
    lib.sv_probe_ex2.argtypes = [P, P, P, I64, P]
    lib.sv_probe_exp1.argtypes = [P, P, P, I64, P]
    assert torch.cuda.is_available()
    return lib


def stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_ex2_polynomial_and_special_function_unit(probe):
    dev = torch.device("cuda:0")
    y = np.concatenate([np.linspace(-126.0, 0.0, 1 << 22, dtype=np.float32),
                        np.float32([0.0, -0.0, -0.5, 0.5 - 1.0, -0.25, -1e-7, -125.5, -126.0]),
                        -np.random.default_rng(0).random(1 << 20, dtype=np.float32) * 3])
    yd = torch.from_numpy(y).to(dev)
    poly = torch.empty_like(yd)
    mufu = torch.empty_like(yd)
    assert probe.sv_probe_ex2(yd.data_ptr(), poly.data_ptr(), mufu.data_ptr(), y.size,
                              stream()) == 0
    torch.cuda.synchronize()
    ref = np.exp2(y.astype(np.float64))
    rel_poly = np.abs(poly.cpu().numpy() / ref - 1.0)
    rel_mufu = np.abs(mufu.cpu().numpy() / ref - 1.0)
    print(f"ex2_poly_x2 max rel {rel_poly.max():.3e}, ex2f max rel {rel_mufu.max():.3e}")
    assert rel_poly.max() <= 2.5e-7
    assert rel_mufu.max() <= 2.0 * 2.0 ** -23


def test_exponential_variates_over_every_uniform(probe):
    dev = torch.device("cuda:0")
    j = np.arange(1 << 23, dtype=np.uint32)
    w = (j << np.uint32(9)) | np.uint32(0x1ff) * (j & np.uint32(1))  # low 9 bits unused
    wd = torch.from_numpy(w.view(np.int32)).to(dev)
    one = torch.empty(w.size, dtype=torch.float32, device=dev)
    two = torch.empty_like(one)
    assert probe.sv_probe_exp1(wd.data_ptr(), one.data_ptr(), two.data_ptr(), w.size,
                               stream()) == 0
    torch.cuda.synchronize()
    e1, e2 = one.cpu().numpy(), two.cpu().numpy()
    np.testing.assert_array_equal(e1.view(np.uint32), e2.view(np.uint32))
    u = (j.astype(np.float64) + 0.5) * 2.0 ** -23
    ref = np.log2(u)
    rel = np.abs(e1 / ref - 1.0)
    series = w >= np.uint32(0xE0000000)
    print(f"series max rel {rel[series].max():.3e}, lg2 max rel {rel[~series].max():.3e}")
    assert rel[series].max() <= 2.0 * 2.0 ** -23
    assert rel[~series].max() <= 1e-6
    assert (e1 < 0).all()  # u' < 1: every variate is a finite negative log

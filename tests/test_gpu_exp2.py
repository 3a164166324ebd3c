"""GPU check of the FP32-pipe polynomial 2^x against the exact value and
against the MUFU ex2.approx it stands in for, over the range the softmax
produces (scores minus the running max: from the clamp at -126 up to the
largest positive argument the lazy max allows) plus the values the mask
produces (-inf).  The probe kernel runs the very device function the
attention kernels inline (tests/gpu_probe/exp2_probe.cu)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out = str(tmp_path_factory.mktemp("probe") / "libexp2_probe.so")
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                           "-Xcompiler", "-fPIC", "-shared", "-o", out,
                           os.path.join(HERE, "gpu_probe", "exp2_probe.cu")])
    lib = ctypes.CDLL(out)
    lib.exp2_probe.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_void_p]
    return lib


def _run(lib, x: np.ndarray):
    dev = torch.device("cuda:0")
    xd = torch.from_numpy(x.astype(np.float32)).to(dev)
    yp, ym = torch.empty_like(xd), torch.empty_like(xd)
    rc = lib.exp2_probe(xd.data_ptr(), yp.data_ptr(), ym.data_ptr(), xd.numel() // 2,
                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    return yp.cpu().double().numpy(), ym.cpu().double().numpy()


def test_poly_error_over_softmax_range(probe):
    x = np.linspace(-125.0, 64.0, 4000000).astype(np.float32)
    yp, ym = _run(probe, x)
    exact = np.exp2(x.astype(np.float64))
    rel_p = yp / exact - 1.0
    rel_m = ym / exact - 1.0
    print(f"poly max rel {np.abs(rel_p).max():.3e} mean {rel_p.mean():.2e}; "
          f"ex2.approx max rel {np.abs(rel_m).max():.3e}")
    assert np.abs(rel_p).max() <= 7.5e-5
    assert abs(rel_p.mean()) <= 1e-5
    # same value as the MUFU to well within bf16 rounding of P (2^-9)
    assert np.abs(yp / ym - 1.0).max() <= 1e-4


def test_poly_matches_cpu_emulation_bitwise(probe):
    from causal_attention_fwd_b200 import exp2_fit

    g = np.random.default_rng(5)
    x = np.concatenate([g.uniform(-130, 10, 200000), g.normal(0, 3, 200000)]).astype(np.float32)
    yp, _ = _run(probe, x)
    emu = exp2_fit.exp2_emulated(x, exp2_fit.fp32_coefficients()).astype(np.float64)
    # fp32 steps in the same order: equal bits except where the CPU's fma
    # emulation double-rounds (rare, one ulp)
    diff = np.abs(yp - emu) / np.maximum(emu, 1e-38)
    assert (diff > 0).mean() < 1e-3 and diff.max() < 2.4e-7


def test_masked_and_tiny_arguments(probe):
    x = np.array([-np.inf, -1e30, -500.0, -127.0, -126.0, -125.0, 0.0, 1.0], np.float32)
    yp, ym = _run(probe, x)
    assert np.all(np.isfinite(yp)) and np.all(yp >= 0)
    assert np.all(yp[:5] <= 2.0 ** -125)  # at or below the clamp: 2^-126, never garbage
    np.testing.assert_allclose(yp[5:], np.exp2(x[5:].astype(np.float64)), rtol=7.5e-5)
    assert ym[0] == 0.0  # the MUFU gives exact 0 for -inf (the kernels' non-polynomial pairs)

"""The FMA-pipe 2^x of the streaming kernel (Cody-Waite reduction and the
Taylor polynomial of e^(f ln 2) through f^6), against exact powers of two
computed in float64 by numpy, beside the special-function unit's ex2.approx
on the same arguments.  The probe is compiled from tests/cuda/exp2_probe.cu
with nvcc for sm_100a."""
import ctypes
import subprocess
from pathlib import Path

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
HERE = Path(__file__).resolve().parent


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    so = tmp_path_factory.mktemp("exp2") / "exp2_probe.so"
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "--expt-relaxed-constexpr", "-shared", "-Xcompiler", "-fPIC",
                    str(HERE / "cuda" / "exp2_probe.cu"), "-o", str(so)], check=True)
    lib = ctypes.CDLL(str(so))
    lib.exp2_probe.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    return lib


def _run(lib, x):
    xd = torch.from_numpy(x).cuda()
    yf, ys = torch.empty_like(xd), torch.empty_like(xd)
    assert lib.exp2_probe(xd.data_ptr(), yf.data_ptr(), ys.data_ptr(), x.size) == 0
    return yf.cpu().numpy(), ys.cpu().numpy()


def test_fma_exp2_matches_exact_powers(probe):
    rng = np.random.default_rng(0)
    x = np.concatenate([-rng.uniform(0, 125, 1 << 20), -rng.uniform(0, 1, 1 << 16),
                        -np.arange(0, 125, dtype=np.float64),          # integers (f = 0)
                        -np.arange(0, 125, dtype=np.float64) - 0.5,    # |f| = 1/2, the widest
                        ]).astype(np.float32)
    yf, ys = _run(probe, x)
    exact = np.exp2(x.astype(np.float64))
    rel_f = np.abs(yf - exact) / exact
    rel_s = np.abs(ys - exact) / exact
    print(f"max relative error: fma {rel_f.max():.3e}, ex2.approx {rel_s.max():.3e}")
    assert rel_f.max() < 4e-7
    assert rel_f.max() < 2.5 * rel_s.max()
    assert np.all(yf[x == 0] == 1.0)


def test_fma_exp2_tails(probe):
    x = np.array([-np.inf, -1e30, -200.0, -127.0, -126.5, -126.0, -125.0, -124.5, 0.0, -0.0],
                 dtype=np.float32)
    yf, _ = _run(probe, x)
    assert np.all(yf[:6] == 0.0)                       # below 2^-125: 0
    assert yf[6] == np.float32(2.0 ** -125)
    assert abs(yf[7] / 2.0 ** -124.5 - 1) < 4e-7
    assert yf[8] == 1.0 and yf[9] == 1.0


def test_float64_exp2_forms_match_exact_powers(probe):
    """The sampling-tree kernel's float64 2^x, in both forms, against numpy's
    float64 exp2 (itself within about an ulp): within 2e-15 relative over the
    arguments the kernel uses (x <= 0), 0 below 2^-1022."""
    probe.exp2d_probe.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    rng = np.random.default_rng(1)
    x = np.concatenate([-rng.uniform(0, 1000, 1 << 18), -rng.uniform(0, 1, 1 << 16),
                        -np.arange(0, 1000, 1 / 16.0), [0.0, -1021.9, -1022.0, -1e9]])
    xd = torch.from_numpy(x).cuda()
    yt, yy = torch.empty_like(xd), torch.empty_like(xd)
    assert probe.exp2d_probe(xd.data_ptr(), yt.data_ptr(), yy.data_ptr(), x.size) == 0
    yt, yy = yt.cpu().numpy(), yy.cpu().numpy()
    exact = np.exp2(x)
    live = x > -1022.0
    for y in (yt, yy):
        rel = np.abs(y[live] - exact[live]) / exact[live]
        print(f"float64 exp2: max relative error {rel.max():.3e}")
        assert rel.max() < 2e-15
        assert np.all(y[~live] == 0.0)

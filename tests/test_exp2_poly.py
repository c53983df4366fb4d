"""The FMA-pipe base-2 exponential used by the prefill softmax
(csrc/fastexp.cuh with the polynomial of csrc/exp2_poly.h).

CPU: the committed coefficients are what the Remez fit produces; the
polynomial's relative error, with every fp32 operation of the device
sequence emulated (round-to-nearest add for the range reduction, fused
multiply-adds for Horner, integer add of n into the exponent field), stays
within 1e-4 of 2^x over the whole argument range a softmax produces, which
is 20x below the bf16 rounding (2^-9) the probabilities get next.

GPU: the device function itself, compiled for sm_100a, against the hardware
approximation ex2.approx.ftz.f32 on the same arguments: the two agree within
the polynomial's bound plus the hardware unit's documented error."""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_kv_cache_408_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly_fit  # noqa: E402

BOUND = 1.0e-4


def header_coeffs():
    text = open(os.path.join(CSRC, "exp2_poly.h")).read()
    vals = {}
    for line in text.splitlines():
        if line.startswith("constexpr float kExp2Poly"):
            name, rhs = line.split("=")
            vals[int(name.split("kExp2Poly")[1])] = np.float32(float(rhs.split("f;")[0]))
    return [vals[j] for j in range(len(vals))]


def emulate(x):
    """The device sequence of exp2_fma2 in fp32, emulated with numpy."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-120.0))
    r = np.float32(12582912.0)
    t = (x + r).astype(np.float32)
    n = (t - r).astype(np.float32)
    f = (x - n).astype(np.float32)
    c = header_coeffs()

    def fma(a, b, cc):  # a*b is exact in fp64; one rounding to fp32 after the add
        return (a.astype(np.float64) * b.astype(np.float64) + np.float64(cc)).astype(np.float32)

    p = fma(np.full_like(f, c[3]), f, c[2])
    p = fma(p, f, c[1])
    p = fma(p, f, c[0])
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_header_matches_the_fit():
    c32, E, E32 = exp2_poly_fit.fit()
    assert open(os.path.join(CSRC, "exp2_poly.h")).read() == exp2_poly_fit.header_text(c32, E, E32)
    assert E < 8e-5 and E32 < 8e-5


def test_reduction_and_polynomial_within_bound():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-120, 10, 2_000_001, dtype=np.float32),
                        rng.uniform(-120, 10, 1_000_000).astype(np.float32),
                        np.arange(-120, 11, dtype=np.float32),              # integers: f = 0
                        np.arange(-120, 10, dtype=np.float32) + 0.5])        # ties of the rounding
    got = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < BOUND, rel.max()


def test_far_negative_and_masked_arguments_give_a_negligible_weight():
    x = np.array([-121.0, -500.0, -1e30, -np.inf], np.float32)
    got = emulate(x)
    assert np.all(got > 0) and np.all(got <= 2.0 ** -119)


def test_a_wrong_coefficient_or_reduction_is_caught(monkeypatch):
    """Planted mistakes: the linear coefficient off by 0.1%, and truncation
    instead of rounding in the reduction (f in [0, 1), outside the fitted
    interval), each push the error past the bound."""
    good = header_coeffs()
    bad = list(good)
    bad[1] = np.float32(bad[1] * 1.001)
    monkeypatch.setattr(sys.modules[__name__], "header_coeffs", lambda: bad)
    x = np.linspace(-20, 8, 100001, dtype=np.float32)
    rel = np.abs(emulate(x) - np.exp2(x.astype(np.float64))) / np.exp2(x.astype(np.float64))
    assert rel.max() > BOUND
    monkeypatch.setattr(sys.modules[__name__], "header_coeffs", lambda: good)
    # truncation: f in [0, 1) is outside the fitted interval
    f = np.linspace(0.5, 1.0, 10001)
    p = np.polyval(np.array(good[::-1], np.float64), f)
    assert (np.abs(p - np.exp2(f)) / np.exp2(f)).max() > BOUND


@pytest.mark.gpu
def test_device_function_agrees_with_the_hardware_exponential(cuda_device, tmp_path):
    """exp2_fma2 compiled for sm_100a against ex2.approx.ftz.f32: within the
    polynomial's bound plus 2^-21 for the hardware unit."""
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    exe = str(tmp_path / "exp2_check")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-I", CSRC,
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "gpu_checks", "exp2_check.cu"),
                    "-o", exe], check=True)
    rng = np.random.default_rng(1)
    x = np.concatenate([np.linspace(-119.5, 9.5, 400_001, dtype=np.float32),
                        rng.uniform(-100, 9, 200_000).astype(np.float32)])
    res = subprocess.run([exe], input=x.tobytes(), capture_output=True, check=True).stdout
    out = np.frombuffer(res, np.float32).reshape(-1, 2).astype(np.float64)
    poly, hw = out[:, 0], out[:, 1]
    assert np.all(hw > 0)
    rel = np.abs(poly - hw) / hw
    assert rel.max() < BOUND + 2.0 ** -21, rel.max()
    # and both against the exact value
    ref = np.exp2(x.astype(np.float64))
    assert (np.abs(poly - ref) / ref).max() < BOUND

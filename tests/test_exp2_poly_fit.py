"""Provenance of the polynomial exponential of the attention softmax.

One pair of exponentials in four runs on the FMA pipe instead of the MUFU:
2^x = 2^j * 2^f with j = round(x) and f in [-1/2, 1/2], where 2^f is a
degree-3 polynomial.  Its coefficients are the minimax fit of 2^f on
[-1/2, 1/2] for relative error, found by the Remez exchange algorithm.  This
test re-derives that fit and checks the library's coefficients against it
and against the error bound, and emulates the whole device routine (range
reduction, Horner steps, exponent add) in float32 over the range the
softmax feeds it."""
import os
import re

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CUH = os.path.join(HERE, "..", "dynamic_sparse_attention_minf_b200", "csrc", "minf_device.cuh")
BOUND = 7.5e-5


def _device_coefficients():
    """c3, c2, c1, c0 of exp2_poly_x2, read from the CUDA source."""
    src = open(CUH).read()
    body = src[src.index("exp2_poly_x2"):]
    body = body[: body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f32x2_pack\(([0-9.]+)f, \1f\)", body)]
    assert len(vals) == 4, vals
    return np.array(vals)


def remez_relative(deg=3, a=-0.5, b=0.5, iters=25, grid=200001):
    """Minimax polynomial (highest power first) for 2^x on [a, b], relative
    error: solve p(x_i) + (-1)^i E 2^x_i = 2^x_i on deg + 2 reference points,
    move the points to the alternating extrema of the error, repeat."""
    n = deg + 2
    x = 0.5 * (a + b) - 0.5 * (b - a) * np.cos(np.pi * np.arange(n) / (n - 1))
    g = np.linspace(a, b, grid)
    for _ in range(iters):
        f = 2.0 ** x
        A = np.vander(x, deg + 1, increasing=True)
        A = np.hstack([A, ((-1.0) ** np.arange(n) * f)[:, None]])
        sol = np.linalg.solve(A, f)
        c = sol[: deg + 1][::-1]
        err = (np.polyval(c, g) - 2.0 ** g) / 2.0 ** g
        ext = [0] + [i for i in range(1, grid - 1) if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [grid - 1]
        pts = []
        for i in ext:
            if pts and np.sign(err[i]) == np.sign(err[pts[-1]]):
                if abs(err[i]) > abs(err[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        while len(pts) > n:
            pts.pop(0 if abs(err[pts[0]]) < abs(err[pts[-1]]) else -1)
        if len(pts) == n:
            x = g[pts]
    return c, float(np.abs(err).max())


def test_coefficients_are_the_minimax_fit():
    c_fit, e_fit = remez_relative()
    c_dev = _device_coefficients()
    assert np.allclose(c_dev, c_fit, rtol=1e-6, atol=0), (c_dev, c_fit)
    g = np.linspace(-0.5, 0.5, 400001)
    e_dev = np.abs((np.polyval(c_dev, g) - 2.0 ** g) / 2.0 ** g).max()
    assert e_fit < BOUND and e_dev < BOUND
    # equioscillation: the fit's error reaches its maximum at both ends
    for end in (-0.5, 0.5):
        assert abs((np.polyval(c_fit, end) - 2.0 ** end) / 2.0 ** end) > 0.999 * e_fit


def test_device_routine_emulated_in_float32():
    """Round-to-integer by adding 1.5 * 2^23, f = x - j, Horner in float32,
    j added to the exponent field; x clamped at -126."""
    c3, c2, c1, c0 = (np.float32(v) for v in _device_coefficients())
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.arange(-125, 9) + 0.5]).astype(np.float32)
    xr = np.maximum(x, np.float32(-126.0))
    k = np.float32(12582912.0)
    t = (xr + k).astype(np.float32)
    j = (t - k).astype(np.float32)
    f = (xr - j).astype(np.float32)
    p = ((((c3 * f + c2).astype(np.float32) * f + c1).astype(np.float32) * f + c0)).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    y = bits.view(np.float32).astype(np.float64)
    rel = np.abs(y - 2.0 ** x.astype(np.float64)) / 2.0 ** x.astype(np.float64)
    assert rel.max() < BOUND + 1e-6, rel.max()


@pytest.mark.gpu
def test_device_exponentials_against_exact():
    """The device polynomial and the MUFU exponential against 2^x in float64
    over [-125, 8], the range the softmax feeds them (arguments are <= 8
    after the running maximum is subtracted; the polynomial clamps at -126)."""
    import torch
    from dynamic_sparse_attention_minf_b200 import minf
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001), torch.arange(-125, 9) + 0.5]).to("cuda")
    yp, ym = minf.minf_selftest_exp2(x)
    torch.cuda.synchronize()
    exact = torch.exp2(x.double())
    rel_poly = ((yp.double() - exact).abs() / exact).max().item()
    rel_mufu = ((ym.double() - exact).abs() / exact).max().item()
    assert rel_poly < BOUND + 1e-6, rel_poly
    assert rel_mufu < 1e-5, rel_mufu
    # below the clamp the polynomial returns a value no larger than 2^-125
    yl, _ = minf.minf_selftest_exp2(torch.tensor([-130.0, -1e30, -float("inf"), 0.0], device="cuda"))
    torch.cuda.synchronize()
    assert (yl[:3] <= 2.0 ** -125).all() and (yl[:3] >= 0).all() and abs(yl[3].item() - 1.0) < BOUND

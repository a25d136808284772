"""Pins of the oracle's Spatial SwiGLU block (GTR article, 方法详解 §2) against
results fixed independently of it: scipy's 2-D correlation and torch's grouped
convolution for the depthwise mixing, brute-force loops on a tiny grid, the
impulse response (which fixes the orientation of the kernel taps), the
identity kernel (which reduces the block to the plain SwiGLU), and exact
values of SiLU."""
import numpy as np
import pytest
import torch
from scipy.signal import correlate2d

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("k,gh,gw", [(3, 5, 7), (3, 1, 6), (5, 6, 4), (3, 1, 1)])
def test_dwconv_matches_scipy_correlate2d(k, gh, gw):
    B, C = 2, 3
    val = _rng(k + gh).standard_normal((B, gh * gw, C))
    w = _rng(gw).standard_normal((k, k, C))
    b = _rng(7).standard_normal(C)
    got = oracle.dwconv2d(val, w, b, gh=gh, gw=gw).reshape(B, gh, gw, C)
    grid = val.reshape(B, gh, gw, C)
    for bi in range(B):
        for c in range(C):
            ref = correlate2d(grid[bi, :, :, c], w[:, :, c], mode="same", boundary="fill") + b[c]
            np.testing.assert_allclose(got[bi, :, :, c], ref, rtol=1e-13, atol=1e-13)


def test_dwconv_matches_torch_grouped_conv():
    B, gh, gw, C = 2, 9, 11, 8
    val = _rng(1).standard_normal((B, gh * gw, C))
    w = _rng(2).standard_normal((3, 3, C))
    b = _rng(3).standard_normal(C)
    inp = torch.from_numpy(val).reshape(B, gh, gw, C).permute(0, 3, 1, 2)
    wt = torch.from_numpy(w).permute(2, 0, 1).unsqueeze(1)          # [C, 1, 3, 3]
    ref = torch.nn.functional.conv2d(inp, wt, torch.from_numpy(b), padding=1, groups=C)
    ref = ref.permute(0, 2, 3, 1).reshape(B, gh * gw, C).numpy()
    np.testing.assert_allclose(oracle.dwconv2d(val, w, b, gh=gh, gw=gw), ref, rtol=1e-12, atol=1e-12)


def test_dwconv_brute_force_loops():
    gh, gw, C = 3, 4, 2
    val = _rng(5).standard_normal((1, gh * gw, C))
    w = _rng(6).standard_normal((3, 3, C))
    ref = np.zeros((1, gh * gw, C))
    for y in range(gh):
        for x in range(gw):
            for c in range(C):
                s = 0.0
                for dy in (-1, 0, 1):
                    for dx in (-1, 0, 1):
                        yy, xx = y + dy, x + dx
                        if 0 <= yy < gh and 0 <= xx < gw:
                            s += w[dy + 1, dx + 1, c] * val[0, yy * gw + xx, c]
                ref[0, y * gw + x, c] = s
    np.testing.assert_allclose(oracle.dwconv2d(val, w, None, gh=gh, gw=gw), ref, rtol=1e-14, atol=1e-14)


def test_impulse_response_is_the_kernel_turned_half_a_turn():
    # a unit value at (y0, x0) reaches out[y0 - i + 1, x0 - j + 1] through tap (i, j)
    gh, gw = 5, 5
    val = np.zeros((1, gh * gw, 1))
    val[0, 2 * gw + 2, 0] = 1.0
    w = np.arange(1.0, 10.0).reshape(3, 3, 1)
    out = oracle.dwconv2d(val, w, None, gh=gh, gw=gw).reshape(gh, gw)
    np.testing.assert_array_equal(out[1:4, 1:4], w[::-1, ::-1, 0])
    assert np.count_nonzero(out) == 9


def test_identity_kernel_gives_the_plain_swiglu():
    B, gh, gw, Cm, C = 2, 4, 3, 6, 5
    x = _rng(8).standard_normal((B, gh * gw, Cm))
    w_in = _rng(9).standard_normal((Cm, 2 * C))
    w_out = _rng(10).standard_normal((C, Cm))
    w = np.zeros((3, 3, C))
    w[1, 1] = 1.0
    xt = torch.from_numpy(x)
    u = xt @ torch.from_numpy(w_in)
    ref = (torch.nn.functional.silu(u[..., :C]) * u[..., C:]) @ torch.from_numpy(w_out)
    got = oracle.sswiglu(x, w_in, w, np.zeros(C), w_out, gh=gh, gw=gw)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_silu_values():
    a = np.array([0.0, 1.0, -1.0, 40.0, -40.0, 800.0, -800.0])
    got = oracle.silu(a)
    assert got[0] == 0.0
    np.testing.assert_allclose(got[1], 1.0 / (1.0 + np.exp(-1.0)), rtol=1e-15)
    np.testing.assert_allclose(got[2], -1.0 / (1.0 + np.e), rtol=1e-15)
    assert got[3] == 40.0 and got[5] == 800.0          # sigmoid rounds to 1
    assert -1e-15 < got[4] < 0 and got[6] == 0.0 and np.all(np.isfinite(got))
    a = np.linspace(-30, 30, 601)
    ref = torch.nn.functional.silu(torch.from_numpy(a)).numpy()
    np.testing.assert_allclose(oracle.silu(a), ref, rtol=1e-14, atol=1e-300)


def test_mix_takes_gate_first_and_value_second():
    # a gate branch of zeros silences the output whatever the value branch holds
    gh, gw, C = 3, 3, 4
    u = _rng(11).standard_normal((1, gh * gw, 2 * C))
    w = _rng(12).standard_normal((3, 3, C))
    z = u.copy()
    z[..., :C] = 0.0
    assert np.all(oracle.sswiglu_mix(z, w, None, gh=gh, gw=gw) == 0.0)
    z = u.copy()
    z[..., C:] = 0.0
    assert np.all(oracle.sswiglu_mix(z, w, None, gh=gh, gw=gw) == 0.0)
    z[..., C:] = 1.0          # a constant value branch in the interior sums the taps
    mid = oracle.sswiglu_mix(z, w, None, gh=gh, gw=gw).reshape(gh, gw, C)[1, 1]
    np.testing.assert_allclose(mid, oracle.silu(u[0, 4, :C]) * w.sum(axis=(0, 1)), rtol=1e-14)

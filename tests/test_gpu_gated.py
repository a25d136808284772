"""Parity of the fused gate + GLA call (gtr_gla_fwd_gated) with the fp64 oracle.

gtr_gla_fwd_gated computes g = logsigmoid(x W_down W_up + b)/tau and the GLA
forward in one call; on the tensor-core path the gate's second half runs
inside the summary kernel.  Every test compares both results, g and y, with
the oracle (g under the gate kernel's own tolerance, y under tests/parity.py),
over the scan orders, both load paths (tensor-map boxes and per-token
gathers), ragged and reversed chunks, a bias, strong decay (exact chunks in
the output kernel), multi-wave segment plans and the two-call fallback.
"""
import dataclasses
import functools

import numpy as np
import pytest
import torch

import oracle
from linear_vision_backbone_b200 import binding, inputs
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

DIRS = ("LR", "RL", "TB", "BT")


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    from linear_vision_backbone_b200 import build
    build.build()
    binding.load()
    binding.set_path("auto")
    yield
    binding.set_path("auto")


def _check_status():
    rc, bits, _ = binding.device_status()
    assert rc == 0 and bits == 0, (rc, bits)


@functools.lru_cache(maxsize=None)
def _data(wl, bias_scale=0.0, bias_mu=0.0):
    d = inputs.make_inputs(wl)
    if bias_scale or bias_mu:
        gen = torch.Generator().manual_seed(wl.seed + 101)
        d["bias"] = torch.randn(wl.H * wl.dk, generator=gen) * bias_scale + bias_mu
    g = oracle.gate(d["x"], d["w_down"], d["w_up"], d["bias"], tau=wl.tau).reshape(
        wl.B, wl.T, wl.H, wl.dk)
    return d, g


@functools.lru_cache(maxsize=None)
def _oracle_y(wl, direction, bias_scale=0.0, bias_mu=0.0):
    d, g = _data(wl, bias_scale, bias_mu)
    return oracle.gla_fwd(d["q"], d["k"], d["v"], g, d["z"], d["w"], gh=wl.gh, gw=wl.gw,
                          direction=direction)


def _run(wl, direction, chunk=64, bias_scale=0.0, bias_mu=0.0):
    d, g_ref = _data(wl, bias_scale, bias_mu)
    dv = {k: v.cuda() for k, v in d.items()}
    packed = binding.gate_pack(dv["w_down"], dv["w_up"], dv["x"].dtype, wl.H, wl.dk)
    y, g = binding.gla_fwd_gated(dv["x"], packed, dv["bias"], dv["q"], dv["k"], dv["v"], dv["z"],
                                 dv["w"], tau=wl.tau, grid_h=wl.gh, grid_w=wl.gw,
                                 direction=direction, chunk=chunk)
    torch.cuda.synchronize()
    got = g.double().cpu().numpy()
    np.testing.assert_allclose(got, g_ref, rtol=1e-5, atol=1e-6)
    assert np.all(got <= 0.0)
    return y, g, dv, packed


def _check(wl, direction, chunk=64, bias_scale=0.0, bias_mu=0.0):
    y, g, dv, packed = _run(wl, direction, chunk, bias_scale, bias_mu)
    assert_close(y, _oracle_y(wl, direction, bias_scale, bias_mu), inputs.DTYPES[wl.dtype],
                 f"{wl.name} {direction}")
    _check_status()
    return y, g, dv, packed


@pytest.mark.parametrize("direction", DIRS)
def test_gated_640_all_directions(direction):
    # 40 x 40 grid: LR / RL by boxes, TB / BT (40 rows per column) by gathers
    _check(inputs.WORKLOADS["640"], direction)


@pytest.mark.parametrize("direction", ("TB", "BT"))
def test_gated_16k_strided_directions(direction):
    # the benchmark's workload and launch configuration
    _check(inputs.WORKLOADS["16k"], direction)


def test_gated_batched_bf16_rotating_directions_with_bias():
    _check(inputs.WORKLOADS["640b8"], "ROTATE", bias_scale=1.0)


@pytest.mark.parametrize("direction", DIRS + ("ROTATE",))
def test_gated_box_loads_every_order(direction):
    # 64 divides gh: every order's chunk (k, v and the rank-16 gate rows) is one box
    wl = inputs.WORKLOADS["640b8"].with_grid(64, 24)
    _check(dataclasses.replace(wl, B=4), direction, bias_scale=0.5)


@pytest.mark.parametrize("direction", DIRS)
def test_gated_ragged_grid(direction):
    # T = 1073: the last chunk is ragged (RL's box starts before token 0); its
    # padding positions must get g = 0, and TB / BT gather per token
    _check(inputs.WORKLOADS["640"].with_grid(37, 29), direction, bias_scale=1.0)


@pytest.mark.parametrize("direction", ("LR", "BT"))
def test_gated_strong_decay(direction):
    # bias -8: g ~ -0.5 per token, in-chunk cumsums far past the factorised
    # range, so the output kernel takes its exact path
    wl = inputs.WORKLOADS["640"].with_grid(64, 8)
    binding.device_status()
    _check(wl, direction, bias_scale=1.0, bias_mu=-8.0)


def test_gated_many_sequences_multi_wave():
    # 64 x 6 sequences: more than two per SM, the multi-wave segment plan
    wl = dataclasses.replace(inputs.WORKLOADS["640"], B=64, gh=8, gw=8, name="640-b64-8x8")
    _check(wl, "RL", bias_scale=0.5)


def test_gated_equals_the_two_calls():
    # the same g and y as gtr_gate_fwd_packed followed by gtr_gla_fwd, up to rounding
    wl = inputs.WORKLOADS["640"]
    y, g, dv, packed = _check(wl, "TB", bias_scale=1.0)
    g2 = binding.gate_fwd_packed(dv["x"], packed, dv["bias"], 16, wl.H, wl.dk, wl.tau)
    y2 = binding.gla_fwd(dv["q"], dv["k"], dv["v"], g2, dv["z"], dv["w"], grid_h=wl.gh,
                         grid_w=wl.gw, direction="TB")
    torch.cuda.synchronize()
    assert float((g - g2).abs().max()) <= 1e-6
    d16 = (y.float() - y2.float()).abs().max()
    assert float(d16) <= 2e-2 * float(y2.float().pow(2).mean().sqrt())


def test_gated_fallback_two_calls():
    # chunk 32 has no tensor-core kernel: the call runs the gate and gtr_gla_fwd
    wl = inputs.WORKLOADS["640"].with_grid(20, 24)
    assert binding.path_for(1, 6, 20, 24, 64, 64, 32, torch.float16) == "simt"
    _check(wl, "BT", chunk=32, bias_scale=1.0)

"""Parity of the token mixer's projections (gtr_mixer_in_proj / gtr_mixer_out_proj)
with the fp64 oracle, alone and chained with the gate and the GLA into the
whole token mixer: x -> (q, k, v, z) -> y -> y W_o.

The projections are plain GEMMs with fp32 accumulation; their outputs are
compared with the fp64 product rounded to the storage dtype under the rules of
tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_vision_backbone_b200 import binding, inputs
from tests.parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    from linear_vision_backbone_b200 import build
    build.build()
    binding.load()


def _weights(dm, n, dtype, seed):
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(dm, n, generator=gen) / dm ** 0.5).to(dtype)


@pytest.mark.parametrize("dtype", (torch.float16, torch.bfloat16))
@pytest.mark.parametrize("B,T,dm,H,dk,dv", [(1, 1600, 384, 6, 64, 64), (2, 77, 128, 3, 32, 64)])
def test_in_projection(dtype, B, T, dm, H, dk, dv):
    gen = torch.Generator().manual_seed(T + dm)
    x = torch.randn(B, T, dm, generator=gen).to(dtype)
    w = _weights(dm, 2 * H * dk + 2 * H * dv, dtype, dm + 1)
    q, k, v, z = binding.mixer_in_proj(x.cuda(), w.cuda(), H, dk, dv)
    torch.cuda.synchronize()
    ref = oracle.linear(x, w)
    cuts = np.cumsum([0, H * dk, H * dk, H * dv, H * dv])
    for t, name, d, a, b in ((q, "q", dk, cuts[0], cuts[1]), (k, "k", dk, cuts[1], cuts[2]),
                             (v, "v", dv, cuts[2], cuts[3]), (z, "z", dv, cuts[3], cuts[4])):
        assert t.shape == (B, T, H, d)
        assert_close(t, ref[..., a:b].reshape(B, T, H, d), dtype, name)


@pytest.mark.parametrize("dtype", (torch.float16, torch.bfloat16))
def test_out_projection(dtype):
    gen = torch.Generator().manual_seed(3)
    y = torch.randn(2, 300, 384, generator=gen).to(dtype)
    w = _weights(384, 384, dtype, 4)
    out = binding.mixer_out_proj(y.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert_close(out, oracle.linear(y, w), dtype, "out")


def test_whole_token_mixer_640():
    # x -> q, k, v, z (in-projection) -> g (gate) -> y (GLA, RMSNorm x SiLU) -> y W_o,
    # every step through the C ABI, against the oracle chain (each step's input the
    # oracle's own previous output rounded to the storage dtype, as the GPU stores it)
    wl = inputs.WORKLOADS["640"]
    d = inputs.make_inputs(wl)
    dt = torch.float16
    H, dk = wl.H, wl.dk
    w_in = _weights(wl.d_model, 4 * H * dk, dt, 11)
    w_o = _weights(H * dk, wl.d_model, dt, 12)
    x = d["x"]
    xd = x.cuda()
    q, k, v, z = binding.mixer_in_proj(xd, w_in.cuda(), H, dk)
    g = binding.gate_fwd(xd, d["w_down"].cuda(), d["w_up"].cuda(), d["bias"].cuda(), H, dk, wl.tau)
    y = binding.gla_fwd(q, k, v, g, z, d["w"].cuda(), grid_h=wl.gh, grid_w=wl.gw, direction="BT")
    out = binding.mixer_out_proj(y.reshape(wl.B, wl.T, H * dk), w_o.cuda())
    torch.cuda.synchronize()

    proj = oracle.linear(x, w_in)
    r16 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dt)
    qr, kr, vr, zr = (r16(proj[..., i * H * dk:(i + 1) * H * dk].reshape(wl.B, wl.T, H, dk)) for i in range(4))
    for t, r, name in ((q, qr, "q"), (k, kr, "k"), (v, vr, "v"), (z, zr, "z")):
        assert_close(t, r.double().numpy(), dt, name)
    gr = oracle.gate(x, d["w_down"], d["w_up"], d["bias"], tau=wl.tau).reshape(wl.B, wl.T, H, dk)
    # the GLA stage on the GPU's own projections (the oracle rounds like the GPU stores)
    yr = oracle.gla_fwd(q.cpu(), k.cpu(), v.cpu(), gr, z.cpu(), d["w"], gh=wl.gh, gw=wl.gw, direction="BT")
    assert_close(y, yr, dt, "y")
    outr = oracle.linear(y.cpu().reshape(wl.B, wl.T, H * dk), w_o)
    assert_close(out, outr, dt, "out")

"""Parity of the Spatial SwiGLU block (gtr_sswiglu_mix / gtr_sswiglu_fwd) with
the fp64 oracle (GTR article, 方法详解 §2).

The mixing kernel reads 16-bit u, computes in fp32 and rounds h once; it is
compared with the oracle's h from the same 16-bit u under the rules of
tests/parity.py.  The whole block is compared stage by stage: u with the fp64
expansion, h with the oracle's mixing of the GPU's u, y with the fp64 product
of the GPU's h (each stage's input the one the GPU stored, as the GPU uses it).
"""
import numpy as np
import pytest
import torch

import oracle
from linear_vision_backbone_b200 import binding
from tests.parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    from linear_vision_backbone_b200 import build
    build.build()
    binding.load()


def _case(B, gh, gw, C, dtype, seed, bias=True):
    gen = torch.Generator().manual_seed(seed)
    u = torch.randn(B, gh * gw, 2 * C, generator=gen).to(dtype)
    w = (torch.randn(3, 3, C, generator=gen) / 3.0).float()
    b = (torch.randn(C, generator=gen) * 0.1).float() if bias else None
    return u, w, b


# shapes: one token; one grid row; one grid column; 5 channel groups of 8 with a
# ragged grid; strips of one row (many strips); strips of 7 rows with a ragged
# last strip; two images
@pytest.mark.parametrize("dtype", (torch.float16, torch.bfloat16))
@pytest.mark.parametrize("B,gh,gw,C", [(1, 1, 1, 8), (1, 1, 17, 16), (1, 17, 1, 16), (3, 5, 7, 40),
                                       (1, 40, 40, 256), (2, 64, 48, 512)])
def test_mix_matches_oracle(dtype, B, gh, gw, C):
    u, w, b = _case(B, gh, gw, C, dtype, gh * 100 + gw + C)
    h = binding.sswiglu_mix(u.cuda(), w.cuda(), b.cuda(), grid_h=gh, grid_w=gw)
    torch.cuda.synchronize()
    assert h.shape == (B, gh * gw, C)
    assert_close(h, oracle.sswiglu_mix(u, w, b, gh=gh, gw=gw), dtype, "h")


@pytest.mark.parametrize("dtype", (torch.float16, torch.bfloat16))
def test_mix_without_bias(dtype):
    u, w, _ = _case(2, 9, 13, 64, dtype, 5, bias=False)
    h = binding.sswiglu_mix(u.cuda(), w.cuda(), None, grid_h=9, grid_w=13)
    torch.cuda.synchronize()
    assert_close(h, oracle.sswiglu_mix(u, w, None, gh=9, gw=13), dtype, "h")


def test_mix_at_the_16k_grid():
    # 128 x 128 tokens, hidden width 1024: the size the block is measured at
    u, w, b = _case(1, 128, 128, 1024, torch.float16, 16)
    h = binding.sswiglu_mix(u.cuda(), w.cuda(), b.cuda(), grid_h=128, grid_w=128)
    torch.cuda.synchronize()
    assert_close(h, oracle.sswiglu_mix(u, w, b, gh=128, gw=128), torch.float16, "h")


def test_identity_kernel_and_zero_bias_give_the_plain_gated_product():
    # the centre tap alone: h = SiLU(gate) * value, element by element (one
    # rounding of an fp32 product of two exact widened inputs)
    u, _, _ = _case(1, 6, 10, 32, torch.float16, 9)
    w = torch.zeros(3, 3, 32)
    w[1, 1] = 1.0
    h = binding.sswiglu_mix(u.cuda(), w.cuda(), torch.zeros(32).cuda(), grid_h=6, grid_w=10)
    torch.cuda.synchronize()
    ud = u.double().numpy()
    assert_close(h, oracle.silu(ud[..., :32]) * ud[..., 32:], torch.float16, "h")


def test_mix_rejects_a_hidden_width_off_the_vector_size():
    u = torch.zeros(1, 4, 24, device="cuda", dtype=torch.float16)
    with pytest.raises(binding.GtrError) as e:
        binding.sswiglu_mix(u, torch.zeros(3, 3, 12, device="cuda"), None, grid_h=2, grid_w=2)
    assert e.value.status == -2


def test_mix_of_an_empty_batch_launches_nothing():
    u = torch.zeros(0, 16, 64, device="cuda", dtype=torch.float16)
    h = binding.sswiglu_mix(u, torch.zeros(3, 3, 32, device="cuda"), None, grid_h=4, grid_w=4)
    assert h.shape == (0, 16, 32)


@pytest.mark.parametrize("dtype", (torch.float16, torch.bfloat16))
@pytest.mark.parametrize("B,gh,gw,dm,C", [(1, 40, 40, 384, 1024), (2, 7, 9, 64, 96)])
def test_block_stage_by_stage(dtype, B, gh, gw, dm, C):
    gen = torch.Generator().manual_seed(dm + C)
    x = torch.randn(B, gh * gw, dm, generator=gen).to(dtype)
    w_in = (torch.randn(dm, 2 * C, generator=gen) / dm ** 0.5).to(dtype)
    w_out = (torch.randn(C, dm, generator=gen) / C ** 0.5).to(dtype)
    cw = (torch.randn(3, 3, C, generator=gen) / 3.0).float()
    cb = (torch.randn(C, generator=gen) * 0.1).float()
    u = torch.empty(B, gh * gw, 2 * C, device="cuda", dtype=dtype)
    h = torch.empty(B, gh * gw, C, device="cuda", dtype=dtype)
    y = binding.sswiglu_fwd(x.cuda(), w_in.cuda(), cw.cuda(), cb.cuda(), w_out.cuda(), grid_h=gh, grid_w=gw,
                            scratch=(u, h))
    torch.cuda.synchronize()
    assert_close(u, oracle.linear(x, w_in), dtype, "u")
    assert_close(h, oracle.sswiglu_mix(u.cpu(), cw, cb, gh=gh, gw=gw), dtype, "h")
    assert_close(y, oracle.linear(h.cpu(), w_out), dtype, "y")


def test_block_end_to_end_fp16():
    # the whole block against the fp64 block on the same 16-bit inputs: the two
    # intermediate roundings of u and h (2^-11 relative each for fp16) stay
    # well inside the 2e-3 relative L2 bound
    gh = gw = 24
    gen = torch.Generator().manual_seed(77)
    x = torch.randn(1, gh * gw, 128, generator=gen).half()
    w_in = (torch.randn(128, 512, generator=gen) / 128 ** 0.5).half()
    w_out = (torch.randn(256, 128, generator=gen) / 16.0).half()
    cw = (torch.randn(3, 3, 256, generator=gen) / 3.0).float()
    cb = (torch.randn(256, generator=gen) * 0.1).float()
    y = binding.sswiglu_fwd(x.cuda(), w_in.cuda(), cw.cuda(), cb.cuda(), w_out.cuda(), grid_h=gh, grid_w=gw)
    torch.cuda.synchronize()
    ref = oracle.sswiglu(x, w_in, cw, cb, w_out, gh=gh, gw=gw)
    got = y.double().cpu().numpy()
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 2e-3

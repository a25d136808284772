"""The stack of GTR blocks on the GPU (gtr_stack_fwd) against the fp64 oracle.

Tolerance.  A stack that keeps its activations in a 16-bit type cannot be
closer to the exact fp64 stack than that storage allows, and a rounding flip
anywhere early (a 1-ulp change where two pipelines add in different orders)
re-draws the rounding of everything after it.  So the bound comes from the
oracle itself: ``oracle.gtr_stack(..., act_dtype=dtype)`` is the exact stack
with every stage's output rounded to the storage type, and its distance E from
the exact stack is the floor of any such pipeline.  The GPU result must lie
within 2 E of the exact stack in relative L2 and within 3 times the oracle's
largest element error per element (measured: perturbing each stage's output
by 2e-6 relative before rounding moves the rounded oracle by about 1.1 E).
"""
import numpy as np
import pytest
import torch

import oracle
from linear_vision_backbone_b200 import binding, build, inputs

pytestmark = pytest.mark.gpu

DT = {"f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    build.build()
    binding.load()


def _run(x, blocks, dtype, gh, gw, H=6, dk=64, dv=64, directions=None, stream=None):
    dt = DT[dtype]
    dev = torch.device("cuda")
    w = binding.stack_weights(blocks, dt, H, dk, dev, stream=stream)
    xd = x.to(dev).contiguous()
    binding.stack_fwd(xd, w, grid_h=gh, grid_w=gw, H=H, dk=dk, dv=dv, dtype=dt, directions=directions,
                      stream=stream)
    torch.cuda.synchronize()
    return xd.double().cpu().numpy(), w


def _check(got, x, blocks, dtype, gh, gw, H=6, directions=None, what=""):
    exact = oracle.gtr_stack(x, blocks, gh=gh, gw=gw, H=H, directions=directions)
    rounded = oracle.gtr_stack(x, blocks, gh=gh, gw=gw, H=H, directions=directions, act_dtype=DT[dtype])
    norm = np.linalg.norm(exact)
    E = np.linalg.norm(rounded - exact) / norm
    emax = np.max(np.abs(rounded - exact))
    rel = np.linalg.norm(got - exact) / norm
    worst = np.max(np.abs(got - exact))
    assert np.all(np.isfinite(got)), what
    assert rel <= 2 * E, f"{what}: rel-L2 {rel:.3e} vs floor {E:.3e}"
    assert worst <= 3 * emax, f"{what}: max |d| {worst:.3e} vs oracle's {emax:.3e}"
    rc, bits, _ = binding.device_status()
    assert rc == 0 and bits == 0, (rc, bits)
    return rel, E


def test_twelve_blocks_fp16():
    # the backbone's depth and widths on a 24x20 grid (480 tokens: 7.5 chunks of 64)
    x, blocks = inputs.make_stack(12, 1, 24, 20, dtype="f16", seed=5)
    got, _ = _run(x, blocks, "f16", 24, 20)
    _check(got, x, blocks, "f16", 24, 20, what="12 blocks f16")


def test_one_block_each_direction_bf16_with_norms_and_bias():
    x, blocks = inputs.make_stack(1, 2, 16, 12, dtype="bf16", seed=6, random_norms=True, bias_std=0.5)
    for d in ("LR", "RL", "TB", "BT"):
        got, _ = _run(x, blocks, "bf16", 16, 12, directions=(d,))
        _check(got, x, blocks, "bf16", 16, 12, directions=(d,), what=f"1 block bf16 {d}")


def test_given_directions_and_graph_replay():
    # four blocks in the reverse rotation, captured into one CUDA graph: a
    # replay equals the direct call bit for bit and both match the oracle
    dirs = ("BT", "TB", "RL", "LR")
    gh, gw, dt = 16, 16, torch.float16
    x, blocks = inputs.make_stack(4, 2, gh, gw, dtype="f16", seed=7, random_norms=True, bias_std=0.3)
    dev = torch.device("cuda")
    s = torch.cuda.Stream()
    w = binding.stack_weights(blocks, dt, 6, 64, dev, stream=s)
    ws = torch.empty(binding.stack_workspace_bytes(2, gh, gw, 384, 6, 64, 64, 1024), device=dev,
                     dtype=torch.uint8)
    x0 = x.to(dev)
    xd = x0.clone()
    kw = dict(grid_h=gh, grid_w=gw, H=6, dk=64, dv=64, dtype=dt, directions=dirs, workspace=ws, stream=s)
    with torch.cuda.stream(s):
        binding.stack_fwd(xd, w, **kw)           # uncaptured first call on the stream
    s.synchronize()
    direct = xd.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        binding.stack_fwd(xd, w, **kw)
    for _ in range(2):
        with torch.cuda.stream(s):
            xd.copy_(x0)
            g.replay()
        s.synchronize()
        assert torch.equal(xd, direct)
    _check(direct.double().cpu().numpy(), x, blocks, "f16", gh, gw, directions=dirs, what="graph f16")
    del g


def test_twelve_blocks_bf16_ragged_grid_norms_and_bias():
    # 13 x 17 = 221 tokens (three chunks and a half), random norm weights and gate bias
    x, blocks = inputs.make_stack(12, 2, 13, 17, dtype="bf16", seed=12, random_norms=True, bias_std=0.5)
    got, _ = _run(x, blocks, "bf16", 13, 17)
    _check(got, x, blocks, "bf16", 13, 17, what="12 blocks bf16 13x17")


def test_full_size_16k_four_blocks():
    # the 128x128 grid (16384 tokens) through LR, RL, TB, BT
    x, blocks = inputs.make_stack(4, 1, 128, 128, dtype="f16", seed=8)
    got, _ = _run(x, blocks, "f16", 128, 128)
    _check(got, x, blocks, "f16", 128, 128, what="16k 4 blocks f16")


def test_residual_path_alone_is_exact():
    # zero output projections: the stack must return x bit for bit
    x, blocks = inputs.make_stack(3, 1, 8, 8, dtype="bf16", seed=9)
    for p in blocks:
        p["w_o"] = torch.zeros_like(p["w_o"])
        p["w_p"] = torch.zeros_like(p["w_p"])
    got, _ = _run(x, blocks, "bf16", 8, 8)
    assert np.array_equal(got, x.double().numpy())


def test_errors_launch_nothing():
    x, blocks = inputs.make_stack(2, 1, 8, 8, dtype="f16", seed=10)
    dev = torch.device("cuda")
    w = binding.stack_weights(blocks, torch.float16, 6, 64, dev)
    xd = x.to(dev)
    before = xd.clone()
    small = torch.empty(1024, device=dev, dtype=torch.uint8)
    with pytest.raises(binding.GtrError) as e:
        binding.stack_fwd(xd, w, grid_h=8, grid_w=8, H=6, dk=64, dv=64, dtype=torch.float16, workspace=small)
    assert e.value.status == -4
    with pytest.raises(binding.GtrError) as e:
        binding.stack_fwd(xd, w, grid_h=8, grid_w=8, H=6, dk=64, dv=64, dtype=torch.float32)
    assert e.value.status == -2
    with pytest.raises(binding.GtrError) as e:                 # dk = 48: no GLA kernel for it
        binding.stack_fwd(xd, w, grid_h=8, grid_w=8, H=8, dk=48, dv=48, dtype=torch.float16)
    assert e.value.status == -2
    torch.cuda.synchronize()
    assert torch.equal(xd, before)

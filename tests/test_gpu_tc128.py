"""The tensor-core kernels for dk = dv = 128 (gla_sum_tc128 / gla_out_tc128)
against the fp64 oracle, through the C ABI.

The scaling sweep's full-size grids run through these kernels in
tests/test_gpu_parity.py; here: every scan order and the per-batch rotation
on ragged grids (the last chunk partly past the sequence), both 16-bit types,
random RMSNorm weights, the chunk states of the summary + scan stages element
by element, chunks whose gate span sends their scores to the exact CUDA-core
sum, and the path selection.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_vision_backbone_b200 import binding, build, inputs
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    build.build()
    binding.load()
    binding.set_path("auto")
    yield
    binding.set_path("auto")


def _run(d, gh, gw, direction, chunk=64):
    dv = {k: v.cuda() for k, v in d.items()}
    y = binding.gla_fwd(dv["q"], dv["k"], dv["v"], dv["g"], dv["z"], dv["w"], grid_h=gh, grid_w=gw,
                        direction=direction, chunk=chunk)
    torch.cuda.synchronize()
    ref = oracle.gla_fwd(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], gh=gh, gw=gw, direction=direction)
    return y, ref


def test_path_selection():
    assert binding.path_for(1, 4, 16, 16, D, D, 64, torch.bfloat16) == "tc"
    assert binding.path_for(1, 4, 16, 16, D, D, 64, torch.float16) == "tc"
    assert binding.path_for(1, 4, 16, 16, D, D, 32, torch.bfloat16) == "simt"
    assert binding.path_for(1, 4, 16, 16, D, D, 64, torch.float32) == "simt"


@pytest.mark.parametrize("dtype", ("f16", "bf16"))
@pytest.mark.parametrize("direction", ("LR", "RL", "TB", "BT", "ROTATE"))
def test_every_order_ragged_grid(dtype, direction):
    gh, gw = 24, 20                      # T = 480: seven chunks and a half
    d = inputs.make_custom(4, 2, gh, gw, D, D, dtype, seed=301, qk_std=D ** -0.5, w_random=True)
    y, ref = _run(d, gh, gw, direction)
    assert_close(y, ref, inputs.DTYPES[dtype], f"d128 {dtype} {direction}")
    rc, bits, _ = binding.device_status()
    assert rc == 0 and bits == 0, (rc, bits)


@pytest.mark.parametrize("gh,gw", [(1, 1), (1, 65), (8, 8), (3, 50)])
def test_small_and_one_chunk_grids(gh, gw):
    d = inputs.make_custom(2, 3, gh, gw, D, D, "bf16", seed=311, qk_std=D ** -0.5)
    for direction in ("LR", "BT"):
        y, ref = _run(d, gh, gw, direction)
        assert_close(y, ref, torch.bfloat16, f"d128 {gh}x{gw} {direction}")


def test_matches_the_simt_kernels():
    gh, gw = 16, 40
    d = inputs.make_custom(1, 4, gh, gw, D, D, "f16", seed=321, qk_std=D ** -0.5)
    y_tc, ref = _run(d, gh, gw, "TB")
    binding.set_path("simt")
    try:
        y_simt, _ = _run(d, gh, gw, "TB")
    finally:
        binding.set_path("auto")
    assert_close(y_tc, ref, torch.float16, "tc")
    assert_close(y_simt, ref, torch.float16, "simt")


@pytest.mark.parametrize("direction,gh,gw", [("LR", 20, 13), ("BT", 20, 13), ("TB", 80, 56)])
def test_chunk_states(direction, gh, gw):
    # 80 x 56: 70 chunks, so the boundary scan holds each range of segments in
    # one long register window
    d = inputs.make_custom(2, 2, gh, gw, D, D, "bf16", seed=331)
    st = binding.chunk_states(d["k"].cuda(), d["v"].cuda(), d["g"].cuda(), grid_h=gh, grid_w=gw,
                              direction=direction, chunk=64)
    ref = oracle.chunk_states(d["k"], d["v"], d["g"], gh=gh, gw=gw, direction=direction, chunk=64)
    got = st.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(ref ** 2)))
    # fp32 accumulation of two-term 16-bit keys against the exact values
    bound = 1e-4 * (np.abs(ref) + rms)
    worst = float(np.max(np.abs(got - ref) / bound))
    assert worst <= 1.0, worst


@pytest.mark.parametrize("dtype", ("f16", "bf16"))
@pytest.mark.parametrize("direction", ("LR", "BT", "ROTATE"))
def test_segments_of_several_chunks(dtype, direction):
    # 8 sequences of 99 chunks (the last one 28 tokens): more chunks than the
    # SMs hold blocks, so every block walks a run of chunks with the state
    # carried on chip from one chunk to the next
    B, H, gh, gw = 2, 4, 90, 70
    dt = inputs.DTYPES[dtype]
    assert binding.segment_chunks(B, H, gh, gw, D, D, 64, dt) > 1
    d = inputs.make_custom(B, H, gh, gw, D, D, dtype, seed=351, qk_std=D ** -0.5, w_random=True)
    y, ref = _run(d, gh, gw, direction)
    assert_close(y, ref, dt, f"d128 segments {dtype} {direction}")
    rc, bits, _ = binding.device_status()
    assert rc == 0 and bits == 0, (rc, bits)


def test_segments_with_exact_chunks_inside():
    # a log-gate span near 20 nats per chunk: some chunks of a segment take the
    # exact scores and carry the state with k^ = k e^{Gam - G}, the others
    # with k~ = k e^{-G}
    B, H, gh, gw = 2, 4, 90, 70
    assert binding.segment_chunks(B, H, gh, gw, D, D, 64, torch.bfloat16) > 1
    d = inputs.make_custom(B, H, gh, gw, D, D, "bf16", seed=361, qk_std=D ** -0.5, g_scale=0.32)
    binding.device_status()
    y, ref = _run(d, gh, gw, "TB")
    assert_close(y, ref, torch.bfloat16, "d128 mixed exact chunks")
    rc, bits, exact = binding.device_status()
    assert rc == 0 and bits == 0
    assert 0 < exact < B * H * 99, exact


def test_strong_decay_takes_the_exact_path():
    # about -12 nats per token: every chunk's span leaves the factorised range
    gh, gw = 16, 16
    d = inputs.make_custom(1, 2, gh, gw, D, D, "f16", seed=341, g_mu=-6.0, g_scale=2.0)
    binding.device_status()
    y, ref = _run(d, gh, gw, "LR")
    assert_close(y, ref, torch.float16, "d128 strong decay")
    rc, bits, exact = binding.device_status()
    assert rc == 0 and bits == 0
    assert exact > 0

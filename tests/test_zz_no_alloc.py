"""The allocation-free entry point gtr_gla_fwd_noalloc against gtr_gla_fwd.

Some callers cannot allocate device memory while they run: a plugin inside an
inference engine that forbids allocation once execution has started, a
real-time loop whose memory footprint is fixed at start-up, a process under a
hard memory cap.  gtr_gla_fwd_noalloc serves them with a fixed static device
scratch array instead of a cudaMalloc'ed workspace.  These tests call it
through the C ABI twice in a row, on different inputs (the scratch keeps the
previous call's contents), and compare each result with gtr_gla_fwd's under
the GPU parity rules of tests/parity.py.  This file is collected last so that
a run stopping at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import pytest
import torch

from linear_vision_backbone_b200 import binding, build, inputs
from tests.parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    build.build()
    binding.load()
    binding.set_path("auto")


def _two_calls(B, H, gh, gw, dk, dv, dtype, direction, chunk, seeds):
    for seed in seeds:
        d = {k: v.cuda() for k, v in
             inputs.make_custom(B, H, gh, gw, dk, dv, dtype, seed=seed, qk_std=dk ** -0.5).items()}
        ref = binding.gla_fwd(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], grid_h=gh, grid_w=gw,
                              direction=direction, chunk=chunk)
        got = binding.gla_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], grid_h=gh,
                                      grid_w=gw, direction=direction, chunk=chunk)
        torch.cuda.synchronize()
        assert_close(got, ref.double().cpu().numpy(), inputs.DTYPES[dtype],
                     f"noalloc {B}x{H} {gh}x{gw} d{dk} {dtype} {direction} seed {seed}")


def test_noalloc_tensor_core_path_two_calls():
    # 640x640-shaped f16 problem on the tcgen05 path, directions differ between calls
    _two_calls(1, 6, 40, 40, 64, 64, "f16", "TB", 64, seeds=(1, 2))
    _two_calls(2, 6, 40, 40, 64, 64, "bf16", "ROTATE", 64, seeds=(3, 4))


def test_noalloc_simt_path_two_calls():
    _two_calls(1, 2, 9, 23, 32, 128, "f32", "BT", 32, seeds=(5, 6))


def test_noalloc_longer_segments_when_states_exceed_scratch():
    # the usual plan for this shape needs more than 8 MiB of boundary states
    B, H, gh, gw, dk = 1, 4, 128, 128, 128
    need = binding.workspace_bytes(B, H, gh, gw, dk, dk, 64, torch.bfloat16)
    assert need > (8 << 20)
    _two_calls(B, H, gh, gw, dk, dk, "bf16", "LR", 64, seeds=(7, 8))


def test_noalloc_rejects_problems_beyond_the_scratch():
    # B*H*(dk*dv + dk)*4 = 128*66048 bytes > 8 MiB: not even one segment per sequence fits
    B, H, dk = 32, 4, 128
    q = torch.zeros(B, 1, H, dk, dtype=torch.float16, device="cuda")
    g = torch.zeros(B, 1, H, dk, dtype=torch.float32, device="cuda")
    with pytest.raises(binding.GtrError) as ei:
        binding.gla_fwd_noalloc(q, q, q, g, q, grid_h=1, grid_w=1)
    assert ei.value.status == -4

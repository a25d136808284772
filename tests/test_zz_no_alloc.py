"""The allocation-free entry point gtr_gla_fwd_noalloc.

Some callers cannot allocate device memory while they run: a plugin inside an
inference engine that forbids allocation once execution has started, a
real-time loop whose memory footprint is fixed at start-up, a process under a
hard memory cap.  gtr_gla_fwd_noalloc serves them with a fixed static device
scratch array instead of a cudaMalloc'ed workspace.  These tests call it
through the C ABI twice in a row, on different inputs (the scratch keeps the
previous call's contents), and compare each result with the fp64 oracle and
with gtr_gla_fwd under the GPU parity rules of tests/parity.py; they run the
plan that falls back to fewer, longer segments when the usual one would not
fit the scratch, on both kernel families; and they check that a call moves
no device memory while gtr_gla_fwd on a new stream does.  This file is
collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import pytest
import torch

import oracle
from linear_vision_backbone_b200 import binding, build, inputs
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

SCRATCH = 8 << 20


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    build.build()
    binding.load()
    binding.set_path("auto")


def _two_calls(B, H, gh, gw, dk, dv, dtype, direction, chunk, seeds):
    dt = inputs.DTYPES[dtype]
    for seed in seeds:
        host = inputs.make_custom(B, H, gh, gw, dk, dv, dtype, seed=seed, qk_std=dk ** -0.5)
        d = {k: v.cuda() for k, v in host.items()}
        ref = oracle.gla_fwd(host["q"], host["k"], host["v"], host["g"], host["z"], host["w"], gh=gh, gw=gw,
                             direction=direction)
        usual = binding.gla_fwd(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], grid_h=gh, grid_w=gw,
                                direction=direction, chunk=chunk)
        got = binding.gla_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], grid_h=gh,
                                      grid_w=gw, direction=direction, chunk=chunk)
        torch.cuda.synchronize()
        what = f"noalloc {B}x{H} {gh}x{gw} d{dk} {dtype} {direction} seed {seed}"
        assert_close(got, ref, dt, what + " vs oracle")
        assert_close(got, usual.double().cpu().numpy(), dt, what + " vs gtr_gla_fwd")
        rc, bits, _ = binding.device_status()
        assert rc == 0 and bits == 0, (rc, bits)


def test_noalloc_tensor_core_path_two_calls():
    # 640x640-shaped f16 problem on the tcgen05 path, directions differ between calls
    _two_calls(1, 6, 40, 40, 64, 64, "f16", "TB", 64, seeds=(1, 2))
    _two_calls(2, 6, 40, 40, 64, 64, "bf16", "ROTATE", 64, seeds=(3, 4))


def test_noalloc_simt_path_two_calls():
    _two_calls(1, 2, 9, 23, 32, 128, "f32", "BT", 32, seeds=(5, 6))


def test_noalloc_longer_segments_when_states_exceed_scratch():
    # the usual plan for this shape needs more than 8 MiB of boundary states
    # (74 segments per sequence); the scratch takes 31, each walking 8-9 chunks
    B, H, gh, gw, dk = 1, 4, 128, 128, 128
    assert binding.workspace_bytes(B, H, gh, gw, dk, dk, 64, torch.bfloat16) > SCRATCH
    _two_calls(B, H, gh, gw, dk, dk, "bf16", "LR", 64, seeds=(7, 8))


def test_noalloc_longer_segments_on_the_tensor_core_path():
    # 384 sequences of 16 chunks: the usual multi-wave plan takes one chunk per
    # segment (about 100 MB of states); the scratch holds one segment per sequence
    B, H, gh, gw = 64, 6, 32, 32
    assert binding.path_for(B, H, gh, gw, 64, 64, 64, torch.float16) == "tc"
    assert binding.workspace_bytes(B, H, gh, gw, 64, 64, 64, torch.float16) > SCRATCH
    assert B * H * (64 * 64 + 64) * 4 + 256 <= SCRATCH
    _two_calls(B, H, gh, gw, 64, 64, "f16", "TB", 64, seeds=(9, 10))


def test_noalloc_d128_tensor_core_path():
    # 64 chunks of one head: 64 x 64 KB of chunk states fit the scratch, so the
    # d = 128 tensor-core kernels run (one chunk per segment)
    B, H, gh, gw = 1, 1, 64, 64
    assert binding.path_for(B, H, gh, gw, 128, 128, 64, torch.bfloat16) == "tc"
    assert binding.workspace_bytes(B, H, gh, gw, 128, 128, 64, torch.bfloat16) <= SCRATCH
    _two_calls(B, H, gh, gw, 128, 128, "bf16", "TB", 64, seeds=(12, 13))


def test_noalloc_rejects_problems_beyond_the_scratch():
    # B*H*(dk*dv + dk)*4 = 128*66048 bytes > 8 MiB: not even one segment per sequence fits
    B, H, dk = 32, 4, 128
    q = torch.zeros(B, 1, H, dk, dtype=torch.float16, device="cuda")
    g = torch.zeros(B, 1, H, dk, dtype=torch.float32, device="cuda")
    with pytest.raises(binding.GtrError) as ei:
        binding.gla_fwd_noalloc(q, q, q, g, q, grid_h=1, grid_w=1)
    assert ei.value.status == -4


def test_noalloc_moves_no_device_memory():
    # Free device memory before and after a call on a stream and a shape the
    # library has not seen: gtr_gla_fwd grows a workspace for a new stream
    # (the control), gtr_gla_fwd_noalloc must leave free memory unchanged.
    B, H, gh, gw = 1, 6, 64, 48
    host = inputs.make_custom(B, H, gh, gw, 64, 64, "f16", seed=11, qk_std=0.125)
    d = {k: v.cuda() for k, v in host.items()}
    out = torch.empty_like(d["v"])
    # the first call of the library on this device places its static arrays
    binding.gla_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], grid_h=gh, grid_w=gw, out=out)
    torch.cuda.synchronize()

    def free_after(fn):
        torch.cuda.synchronize()
        before = torch.cuda.mem_get_info()[0]
        fn()
        torch.cuda.synchronize()
        return before - torch.cuda.mem_get_info()[0]

    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    grown = free_after(lambda: binding.gla_fwd(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], grid_h=gh,
                                               grid_w=gw, out=out, stream=s1))
    assert grown >= (1 << 20), grown          # the measurement sees a workspace allocation
    used = free_after(lambda: binding.gla_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"],
                                                      grid_h=gh, grid_w=gw, out=out, stream=s2))
    assert used == 0, used

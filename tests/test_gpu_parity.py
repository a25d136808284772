"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Every test runs the library on a B200 and compares, element by element, with
the oracle on the same seeded inputs, under the rules of tests/parity.py.
Workloads: the five of linear_vision_backbone_b200.inputs at full size (the
launch configuration the benchmark times), plus ragged, degenerate and
extreme-gate cases.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
from linear_vision_backbone_b200 import binding, inputs
from tests.parity import assert_close, compare

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


def _dev(t):
    return t.cuda() if t is not None else None


@functools.lru_cache(maxsize=None)
def _workload_data(name, grid=None):
    wl = inputs.WORKLOADS[name]
    if grid is not None:
        wl = wl.with_grid(grid)
    return wl, inputs.make_inputs(wl)


@functools.lru_cache(maxsize=None)
def _oracle_gate(name, grid=None):
    wl, d = _workload_data(name, grid)
    return oracle.gate(d["x"], d["w_down"], d["w_up"], d["bias"], tau=wl.tau).reshape(
        wl.B, wl.T, wl.H, wl.dk)


@functools.lru_cache(maxsize=None)
def _oracle_y(name, direction, grid=None):
    wl, d = _workload_data(name, grid)
    g = _oracle_gate(name, grid) if wl.recipe == "proj" else d["g"]
    return oracle.gla_fwd(d["q"], d["k"], d["v"], g, d["z"], d["w"], gh=wl.gh, gw=wl.gw,
                          direction=direction)


def _gpu_step(wl, d, direction, chunk=None):
    """The whole hot path on the GPU: gate projection (when the workload has
    one) then the GLA forward, both through the C ABI."""
    dv = {k: _dev(v) for k, v in d.items()}
    if wl.recipe == "proj":
        g = binding.gate_fwd(dv["x"], dv["w_down"], dv["w_up"], dv["bias"], wl.H, wl.dk, wl.tau)
    else:
        g = dv["g"]
    y = binding.gla_fwd(dv["q"], dv["k"], dv["v"], g, dv["z"], dv["w"], grid_h=wl.gh, grid_w=wl.gw,
                        direction=direction, chunk=chunk or wl.chunk)
    torch.cuda.synchronize()
    return y, g


def _check_status():
    rc, bits, _ = binding.device_status()
    assert rc == 0 and bits == 0, (rc, bits)


def test_tiny_fp32():
    wl, d = _workload_data("tiny")
    y, _ = _gpu_step(wl, d, "LR")
    assert_close(y, _oracle_y("tiny", "LR"), torch.float32, "tiny")
    _check_status()


def test_tiny_fp32_against_stored_oracle_values():
    import json
    import os
    doc = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")))
    stored = np.array([float.fromhex(v) for v in doc["y"]]).reshape(doc["shape"])
    wl, d = _workload_data("tiny")
    y, _ = _gpu_step(wl, d, "LR")
    assert_close(y, stored, torch.float32, "tiny vs stored")


def test_gate_projection_640():
    wl, d = _workload_data("640")
    g = binding.gate_fwd(_dev(d["x"]), _dev(d["w_down"]), _dev(d["w_up"]), _dev(d["bias"]),
                         wl.H, wl.dk, wl.tau)
    ref = _oracle_gate("640")
    got = g.double().cpu().numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6)
    assert np.all(got <= 0.0)


def test_gate_projection_bf16_with_bias():
    gen = torch.Generator().manual_seed(11)
    x = torch.randn(3, 100, 384, generator=gen).to(torch.bfloat16)
    wd = torch.randn(384, 16, generator=gen) / 384 ** 0.5
    wu = torch.randn(16, 6 * 64, generator=gen) / 4
    b = torch.randn(6 * 64, generator=gen) * 2
    g = binding.gate_fwd(x.cuda(), wd.cuda(), wu.cuda(), b.cuda(), 6, 64, 16.0)
    ref = oracle.gate(x, wd, wu, b, tau=16.0).reshape(3, 100, 6, 64)
    np.testing.assert_allclose(g.double().cpu().numpy(), ref, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("dtype,B,T,dm,H,bias", [
    (torch.float16, 1, 1600, 384, 6, False),    # the 640x640 workload's shapes
    (torch.bfloat16, 3, 100, 384, 6, True),     # bf16 x, three W_down terms, bias
    (torch.float16, 1, 5, 64, 1, True),         # fewer tokens than one tile, smallest width
    (torch.float16, 2, 777, 192, 7, True),      # ragged last tile, H*dk = 448 (the largest)
])
def test_gate_packed_weights(dtype, B, T, dm, H, bias):
    # the tensor-core gate with weights packed once: against the oracle, and identical to
    # gtr_gate_fwd (which packs per call and runs the same kernels)
    gen = torch.Generator().manual_seed(T + dm)
    x = torch.randn(B, T, dm, generator=gen).to(dtype)
    wd = torch.randn(dm, 16, generator=gen) / dm ** 0.5
    wu = torch.randn(16, H * 64, generator=gen) / 4
    b = torch.randn(H * 64, generator=gen) if bias else None
    xd, wdd, wud = x.cuda(), wd.cuda(), wu.cuda()
    bd = b.cuda() if bias else None
    packed = binding.gate_pack(wdd, wud, dtype, H, 64)
    g = binding.gate_fwd_packed(xd, packed, bd, 16, H, 64, 16.0)
    g2 = binding.gate_fwd(xd, wdd, wud, bd, H, 64, 16.0)
    ref = oracle.gate(x, wd, wu, b, tau=16.0).reshape(B, T, H, 64)
    np.testing.assert_allclose(g.double().cpu().numpy(), ref, rtol=1e-5, atol=1e-6)
    assert torch.equal(g, g2)
    assert np.all(g.cpu().numpy() <= 0.0)


@pytest.mark.parametrize("rank,H,dk,dm", [(24, 6, 64, 384), (16, 3, 5, 100), (7, 2, 64, 300)])
def test_gate_projection_other_shapes(rank, H, dk, dm):
    # shapes outside the register-tiled kernel (rank > 16, H*dk not a multiple of 4) and a
    # model width that is not a multiple of the staging slab
    gen = torch.Generator().manual_seed(rank)
    x = torch.randn(2, 77, dm, generator=gen).to(torch.float16)
    wd = torch.randn(dm, rank, generator=gen) / dm ** 0.5
    wu = torch.randn(rank, H * dk, generator=gen) / rank ** 0.5
    b = torch.randn(H * dk, generator=gen)
    g = binding.gate_fwd(x.cuda(), wd.cuda(), wu.cuda(), b.cuda(), H, dk, 4.0)
    ref = oracle.gate(x, wd, wu, b, tau=4.0).reshape(2, 77, H, dk)
    np.testing.assert_allclose(g.double().cpu().numpy(), ref, rtol=1e-5, atol=2e-6)


@pytest.mark.parametrize("direction", DIRS)
def test_640_all_directions(direction):
    wl, d = _workload_data("640")
    y, _ = _gpu_step(wl, d, direction)
    assert_close(y, _oracle_y("640", direction), torch.float16, f"640 {direction}")
    _check_status()


def test_640_batched_bf16_rotating_directions():
    wl, d = _workload_data("640b8")
    y, _ = _gpu_step(wl, d, "ROTATE")
    assert_close(y, _oracle_y("640b8", "ROTATE"), torch.bfloat16, "640b8")
    _check_status()


@pytest.mark.parametrize("direction", ("TB", "BT"))
def test_16k_strided_directions(direction):
    wl, d = _workload_data("16k")
    y, _ = _gpu_step(wl, d, direction)
    assert_close(y, _oracle_y("16k", direction), torch.float16, f"16k {direction}")
    _check_status()


@pytest.mark.parametrize("grid", inputs.SWEEP_GRIDS)
def test_scaling_sweep_bf16_d128(grid):
    wl, d = _workload_data("sweep", grid)
    y, _ = _gpu_step(wl, d, "LR")
    assert_close(y, _oracle_y("sweep", "LR", grid), torch.bfloat16, f"sweep {grid}")
    _check_status()


def _run_custom(d, gh, gw, direction, chunk, dtype):
    dv = {k: _dev(v) for k, v in d.items()}
    y = binding.gla_fwd(dv["q"], dv["k"], dv["v"], dv["g"], dv["z"], dv["w"], grid_h=gh, grid_w=gw,
                        direction=direction, chunk=chunk)
    torch.cuda.synchronize()
    ref = oracle.gla_fwd(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], gh=gh, gw=gw,
                         direction=direction)
    return y, ref


@pytest.mark.parametrize("chunk", (16, 32, 64, 128))
@pytest.mark.parametrize("direction", DIRS)
def test_chunk_length_invariance_ragged_grid(chunk, direction):
    gh, gw = 37, 29                                   # T = 1073: ragged for every chunk length
    d = inputs.make_custom(2, 3, gh, gw, 64, 64, "f16", seed=21)
    y, ref = _run_custom(d, gh, gw, direction, chunk, torch.float16)
    assert_close(y, ref, torch.float16, f"chunk {chunk} {direction}")


@pytest.mark.parametrize("path", ("simt", "auto"))
@pytest.mark.parametrize("dtype", ("f16", "bf16"))
def test_both_kernel_families(path, dtype):
    gh, gw = 24, 40
    d = inputs.make_custom(2, 4, gh, gw, 64, 64, dtype, seed=31, w_random=True)
    binding.set_path(path)
    try:
        y, ref = _run_custom(d, gh, gw, "TB", 64, inputs.DTYPES[dtype])
    finally:
        binding.set_path("auto")
    assert_close(y, ref, inputs.DTYPES[dtype], f"{path} {dtype}")


@pytest.mark.parametrize("dk,dv,dtype", [(16, 16, "f32"), (32, 128, "bf16"), (128, 16, "f32"),
                                         (64, 32, "f16"), (128, 128, "f16")])
def test_head_dim_combinations(dk, dv, dtype):
    gh, gw = 9, 23
    d = inputs.make_custom(2, 2, gh, gw, dk, dv, dtype, seed=41, qk_std=dk ** -0.5)
    for direction in ("LR", "BT"):
        y, ref = _run_custom(d, gh, gw, direction, 32, inputs.DTYPES[dtype])
        assert_close(y, ref, inputs.DTYPES[dtype], f"{dk}x{dv} {dtype} {direction}")


@pytest.mark.parametrize("gh,gw", [(1, 1), (1, 5), (3, 1), (2, 3)])
def test_tiny_and_degenerate_grids(gh, gw):
    for dtype in ("f32", "f16"):
        d = inputs.make_custom(3, 2, gh, gw, 64, 64, dtype, seed=51)
        for direction in DIRS:
            y, ref = _run_custom(d, gh, gw, direction, 16, inputs.DTYPES[dtype])
            assert_close(y, ref, inputs.DTYPES[dtype], f"{gh}x{gw} {dtype} {direction}")


def test_strong_decay_takes_the_exact_path():
    # logsigmoid(N(-6, 1)) * 2 ~ -12 nats per token: the decay across one chunk
    # far exceeds what a scaled operand can hold, so the tensor-core kernels
    # must switch those chunks to the exact evaluation.
    gh, gw = 16, 16
    d = inputs.make_custom(1, 2, gh, gw, 64, 64, "f16", seed=61, g_mu=-6.0, g_scale=2.0)
    binding.device_status()
    y, ref = _run_custom(d, gh, gw, "LR", 64, torch.float16)
    assert_close(y, ref, torch.float16, "strong decay")
    rc, bits, exact = binding.device_status()
    assert rc == 0 and bits == 0
    if binding.path_for(1, 2, gh, gw, 64, 64, 64, torch.float16) == "tc":
        assert exact > 0


@pytest.mark.parametrize("dtype", ("f16", "bf16"))
@pytest.mark.parametrize("direction", DIRS + ("ROTATE",))
def test_box_loaded_chunks_every_order(dtype, direction):
    # 64 divides gh, so every scan order's chunk of one head is a single
    # tensor-map box: the token order for LR / RL, a grid column for TB / BT
    # (reversed orders walk the box backwards).  B = 4 gives ROTATE all four.
    gh, gw = 64, 24
    d = inputs.make_custom(4, 2, gh, gw, 64, 64, dtype, seed=23, w_random=True)
    y, ref = _run_custom(d, gh, gw, direction, 64, inputs.DTYPES[dtype])
    assert_close(y, ref, inputs.DTYPES[dtype], f"boxes {dtype} {direction}")
    _check_status()


@pytest.mark.parametrize("dtype", ("f16", "bf16"))
def test_ragged_reversed_box(dtype):
    # RL over T = 1073: the last chunk's box starts before token 0 and reads zeros there
    gh, gw = 37, 29
    d = inputs.make_custom(2, 3, gh, gw, 64, 64, dtype, seed=27)
    y, ref = _run_custom(d, gh, gw, "RL", 64, inputs.DTYPES[dtype])
    assert_close(y, ref, inputs.DTYPES[dtype], f"ragged RL {dtype}")
    _check_status()


@pytest.mark.parametrize("direction", ("RL", "BT"))
def test_strong_decay_reversed_boxes(direction):
    # exact chunks read the staged q, k backwards and rewrite the gate cumsum in scan order
    gh, gw = 64, 4
    d = inputs.make_custom(1, 2, gh, gw, 64, 64, "bf16", seed=63, g_mu=-6.0, g_scale=2.0)
    binding.device_status()
    y, ref = _run_custom(d, gh, gw, direction, 64, torch.bfloat16)
    assert_close(y, ref, torch.bfloat16, f"strong decay {direction}")
    rc, bits, exact = binding.device_status()
    assert rc == 0 and bits == 0
    if binding.path_for(1, 2, gh, gw, 64, 64, 64, torch.bfloat16) == "tc":
        assert exact > 0


@pytest.mark.parametrize("B,H,gh,gw", [(4, 80, 8, 8), (2, 160, 16, 16), (1, 320, 64, 2)])
def test_many_sequences_multi_wave(B, H, gh, gw):
    # more (image, head) sequences than two per SM: the segment plan goes
    # multi-wave and the output CTAs' second chains idle wherever a sequence
    # has an odd number of segments
    d = inputs.make_custom(B, H, gh, gw, 64, 64, "f16", seed=29, qk_std=0.5)
    y, ref = _run_custom(d, gh, gw, "BT", 64, torch.float16)
    assert_close(y, ref, torch.float16, f"{B}x{H} {gh}x{gw}")
    _check_status()


def test_zero_gate_long_memory():
    gh, gw = 64, 64
    d = inputs.make_custom(1, 2, gh, gw, 64, 64, "bf16", seed=71, qk_std=0.125)
    d["g"] = torch.zeros_like(d["g"])
    y, ref = _run_custom(d, gh, gw, "TB", 64, torch.bfloat16)
    assert_close(y, ref, torch.bfloat16, "g = 0")


def _states_close(st, ref):
    """fp32 chunk-boundary states against the fp64 oracle, element by element:
    |got - ref| <= 1e-4 (|ref| + RMS(ref)).  The states are sums of fp32
    products over up to a few thousand tokens; the tensor-core summary's key
    operand carries 22 (fp16 terms) or 16 (bf16 terms) significant bits, so
    its per-element error stays well inside 1e-4 of the state's scale."""
    got = st.double().cpu().numpy()
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got))
    rms = float(np.sqrt(np.mean(ref ** 2)))
    bound = 1e-4 * (np.abs(ref) + rms)
    worst = float(np.max(np.abs(got - ref) / bound))
    assert worst <= 1.0, worst


@pytest.mark.parametrize("chunk", (16, 64, 128))
@pytest.mark.parametrize("direction", ("LR", "BT"))
def test_chunk_states_against_oracle(chunk, direction):
    gh, gw = 20, 13
    d = inputs.make_custom(2, 2, gh, gw, 64, 64, "f16", seed=81)
    st = binding.chunk_states(_dev(d["k"]), _dev(d["v"]), _dev(d["g"]), grid_h=gh, grid_w=gw,
                              direction=direction, chunk=chunk)
    ref = oracle.chunk_states(d["k"], d["v"], d["g"], gh=gh, gw=gw, direction=direction, chunk=chunk)
    _states_close(st, ref)


def test_chunk_states_many_segments():
    # 320 chunks: the boundary scan splits each element's segments into ranges
    # longer than it keeps in registers and re-reads them for its second pass
    gh, gw = 64, 80
    d = inputs.make_custom(1, 2, gh, gw, 64, 64, "bf16", seed=83)
    st = binding.chunk_states(_dev(d["k"]), _dev(d["v"]), _dev(d["g"]), grid_h=gh, grid_w=gw,
                              direction="TB", chunk=16)
    ref = oracle.chunk_states(d["k"], d["v"], d["g"], gh=gh, gw=gw, direction="TB", chunk=16)
    _states_close(st, ref)


def test_chunk_states_into_a_16_byte_aligned_buffer():
    # the summary kernel writes whole 32-byte sectors when its state buffer
    # allows it; a caller's buffer that is only 16-byte aligned takes 16-byte stores
    import ctypes
    gh, gw = 64, 4
    B, H = 1, 2
    d = inputs.make_custom(B, H, gh, gw, 64, 64, "f16", seed=85)
    k, v, g = _dev(d["k"]), _dev(d["v"]), _dev(d["g"])
    nc = gh * gw // 64
    n = B * H * nc * 64 * 64
    buf = torch.full((n + 8,), 3.0, dtype=torch.float32, device="cuda")
    view = buf[4:4 + n]                     # 16 bytes past a 256-byte boundary
    assert view.data_ptr() % 32 == 16
    rc = binding.load().gtr_gla_chunk_states(
        ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(g.data_ptr()),
        ctypes.c_void_p(view.data_ptr()), B, H, gh, gw, 64, 64, 2, 64, 1,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert float(buf[:4].sub(3.0).abs().max()) == 0.0 and float(buf[4 + n:].sub(3.0).abs().max()) == 0.0
    ref = binding.chunk_states(k, v, g, grid_h=gh, grid_w=gw, direction="TB", chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(view.view_as(ref), ref)


@pytest.mark.parametrize("guard", (4096, 4104))
def test_output_stays_inside_its_buffer_and_inputs_untouched(guard):
    # guard 4104 fp16 elements: `out` is 16-byte but not 32-byte aligned (the
    # output kernel's 32-byte row stores then fall back to 16-byte ones)
    gh, gw = 11, 13
    B, H, dk, dv = 2, 3, 64, 64
    d = inputs.make_custom(B, H, gh, gw, dk, dv, "f16", seed=91)
    n = B * gh * gw * H * dv
    for path, chunk in (("simt", 32), ("auto", 32), ("auto", 64)):
        binding.set_path(path)
        try:
            buf = torch.full((n + 2 * guard,), 7.0, dtype=torch.float16, device="cuda")
            out = buf[guard:guard + n].view(B, gh * gw, H, dv)
            dv_ = {k: _dev(v) for k, v in d.items()}
            before = {k: v.clone() for k, v in dv_.items()}
            binding.gla_fwd(dv_["q"], dv_["k"], dv_["v"], dv_["g"], dv_["z"], dv_["w"], grid_h=gh,
                            grid_w=gw, direction="RL", chunk=chunk, out=out)
            torch.cuda.synchronize()
        finally:
            binding.set_path("auto")
        assert torch.all(buf[:guard] == 7.0) and torch.all(buf[guard + n:] == 7.0)
        for k in before:
            assert torch.equal(before[k], dv_[k]), k
        ref = oracle.gla_fwd(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], gh=gh, gw=gw,
                             direction="RL")
        assert_close(out, ref, torch.float16, path)


def test_registered_workspace_too_small_then_large_enough():
    # a caller-registered workspace that is too small is reported (no launch, status -4)
    # and one of exactly gtr_gla_workspace_bytes serves the call; releasing it returns
    # the library to its own buffers
    gh, gw = 40, 40
    d = inputs.make_custom(1, 6, gh, gw, 64, 64, "f16", seed=97)
    dv = {k: _dev(v) for k, v in d.items()}
    args = (dv["q"], dv["k"], dv["v"], dv["g"], dv["z"], dv["w"])
    ref = binding.gla_fwd(*args, grid_h=gh, grid_w=gw, direction="TB")
    need = binding.workspace_bytes(1, 6, gh, gw, 64, 64, 64, torch.float16)
    assert need > 256
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    exact = torch.empty(need, dtype=torch.uint8, device="cuda")
    try:
        binding.set_workspace(small)
        with pytest.raises(binding.GtrError) as ei:
            binding.gla_fwd(*args, grid_h=gh, grid_w=gw, direction="TB")
        assert ei.value.status == -4
        binding.set_workspace(exact)
        y = binding.gla_fwd(*args, grid_h=gh, grid_w=gw, direction="TB")
        torch.cuda.synchronize()
    finally:
        binding.set_workspace(None)
    assert torch.equal(y, ref)
    y2 = binding.gla_fwd(*args, grid_h=gh, grid_w=gw, direction="TB")
    torch.cuda.synchronize()
    assert torch.equal(y2, ref)
    _check_status()


def test_empty_problem_and_argument_errors():
    e = torch.empty(0, 40 * 40, 6, 64, dtype=torch.float16, device="cuda")
    g = torch.empty(0, 40 * 40, 6, 64, dtype=torch.float32, device="cuda")
    y = binding.gla_fwd(e, e, e, g, e, grid_h=40, grid_w=40)
    assert y.shape == e.shape
    # a tensor that starts 2 bytes past a 16-byte boundary
    base = torch.zeros(1 + 1 * 16 * 2 * 64, dtype=torch.float16, device="cuda")
    mis = base[1:].view(1, 16, 2, 64)
    ok = torch.zeros(1, 16, 2, 64, dtype=torch.float16, device="cuda")
    gg = torch.zeros(1, 16, 2, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(binding.GtrError) as ei:
        binding.gla_fwd(mis, ok, ok, gg, ok, grid_h=4, grid_w=4)
    assert ei.value.status == -3
    _check_status()

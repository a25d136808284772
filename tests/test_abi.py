"""The C ABI library loads and exports every entry point of include/gtr_gla.h.

CPU only: no call here launches work or touches a device.  Argument checks
run before any CUDA call, so invalid arguments are rejected on any machine.
"""
import ctypes
import os
import re
import subprocess

import pytest

from linear_vision_backbone_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gtr_gla.h")


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GTR_API\s+[^;(]*?\b(gtr_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def test_header_declares_the_abi():
    syms = header_symbols()
    assert set(syms) == set(binding.EXPORTS), syms


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for s in header_symbols():
        assert s in exported, s
        assert getattr(lib, s) is not None
    # nothing else leaks out of the library
    assert {s for s in exported if s.startswith("gtr_")} == set(header_symbols())


def test_version_and_status_strings(lib):
    assert lib.gtr_abi_version() == 1
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.gtr_status_string(code)
    assert lib.gtr_status_string(12345) == b"unknown status"


def test_invalid_arguments_rejected_before_any_launch(lib):
    P = ctypes.c_void_p(16)
    S = None
    # bad direction, bad dtype, negative sizes, unsupported head dim / chunk
    assert lib.gtr_gla_fwd(P, P, P, P, P, None, P, 1, 1, 4, 4, 64, 64, 7, 64, 1, S) == -1
    assert lib.gtr_gla_fwd(P, P, P, P, P, None, P, 1, 1, 4, 4, 64, 64, 0, 64, 3, S) == -1
    assert lib.gtr_gla_fwd(P, P, P, P, P, None, P, -1, 1, 4, 4, 64, 64, 0, 64, 1, S) == -1
    assert lib.gtr_gla_fwd(P, P, P, P, P, None, P, 1, 1, 4, 4, 48, 64, 0, 64, 1, S) == -2
    assert lib.gtr_gla_fwd(P, P, P, P, P, None, P, 1, 1, 4, 4, 64, 64, 0, 100, 1, S) == -2
    # grid too large for an int
    assert lib.gtr_gla_fwd(P, P, P, P, P, None, P, 1, 1, 65536, 65536, 64, 64, 0, 64, 1, S) == -1
    # empty problems succeed without touching pointers or the device
    assert lib.gtr_gla_fwd(None, None, None, None, None, None, None, 0, 6, 40, 40, 64, 64, 0, 64, 1, S) == 0
    assert lib.gtr_gla_fwd(None, None, None, None, None, None, None, 1, 6, 0, 40, 64, 64, 0, 64, 1, S) == 0
    # gate: bad rank, tau, dtype; rank above the limit is unsupported
    assert lib.gtr_gate_fwd(P, 1, P, P, None, P, 1, 4, 384, 0, 6, 64, 16.0, S) == -1
    assert lib.gtr_gate_fwd(P, 1, P, P, None, P, 1, 4, 384, 16, 6, 64, 0.0, S) == -1
    assert lib.gtr_gate_fwd(P, 5, P, P, None, P, 1, 4, 384, 16, 6, 64, 16.0, S) == -1
    assert lib.gtr_gate_fwd(P, 1, P, P, None, P, 1, 4, 384, 65, 6, 64, 16.0, S) == -2
    assert lib.gtr_gate_fwd(None, 1, None, None, None, None, 0, 4, 384, 16, 6, 64, 16.0, S) == 0
    # packed gate: shapes outside the tensor-core kernel, NULL buffers, short buffers
    nb = lib.gtr_gate_packed_bytes()
    assert nb > 0 and nb % 16 == 0
    assert lib.gtr_gate_pack(P, P, 1, 384, 8, 6, 64, P, nb, S) == -2       # rank 8
    assert lib.gtr_gate_pack(P, P, 1, 100, 16, 6, 64, P, nb, S) == -2      # d_model % 64
    assert lib.gtr_gate_pack(P, P, 0, 384, 16, 6, 64, P, nb, S) == -2      # fp32 x
    assert lib.gtr_gate_pack(P, P, 1, 384, 16, 8, 64, P, nb, S) == -2      # H*dk > 448
    assert lib.gtr_gate_pack(None, P, 1, 384, 16, 6, 64, P, nb, S) == -1
    assert lib.gtr_gate_pack(P, P, 1, 384, 16, 6, 64, P, nb - 16, S) == -4
    assert lib.gtr_gate_fwd_packed(P, 1, P, None, P, 1, 4, 384, 16, 6, 64, 0.0, S) == -1
    assert lib.gtr_gate_fwd_packed(P, 2, P, None, P, 1, 4, 384, 16, 6, 48, 16.0, S) == -2
    assert lib.gtr_gate_fwd_packed(None, 1, P, None, P, 1, 4, 384, 16, 6, 64, 16.0, S) == -1
    assert lib.gtr_gate_fwd_packed(None, 1, None, None, None, 0, 4, 384, 16, 6, 64, 16.0, S) == 0
    assert lib.gtr_gla_set_path(9) == -1
    assert lib.gtr_gla_workspace_bytes(1, 1, 4, 4, 48, 64, 64, 1) == ctypes.c_size_t(-1).value
    assert lib.gtr_gla_workspace_bytes(0, 6, 40, 40, 64, 64, 64, 1) == 0


def test_binding_refuses_a_missing_library(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        # a fresh loader pointed at a path with no library fails loudly
        saved = binding._lib
        binding._lib = None
        try:
            binding.load(str(tmp_path / "nope.so"))
        finally:
            binding._lib = saved


def test_gated_call_rejects_invalid_arguments_before_any_launch(lib):
    P = ctypes.c_void_p(16)
    S = None
    F = ctypes.c_float

    def call(x=P, xdt=1, packed=P, bias=None, dm=384, rank=16, tau=16.0, q=P, g=P, out=P, B=1, H=6,
             gh=8, gw=8, dk=64, dv=64, dir_=0, chunk=64, dtype=1):
        return lib.gtr_gla_fwd_gated(x, xdt, packed, bias, dm, rank, F(tau), q, P, P, P, None, g, out,
                                     B, H, gh, gw, dk, dv, dir_, chunk, dtype, S)

    assert call(dir_=9) == -1                       # GLA arguments as gtr_gla_fwd
    assert call(dk=48) == -2
    assert call(tau=0.0) == -1                      # gate arguments as gtr_gate_fwd_packed
    assert call(xdt=7) == -1
    assert call(rank=8) == -2                       # only the packed (tensor-core) gate shapes
    assert call(dm=100) == -2
    assert call(xdt=0) == -2                        # fp32 x has no packed weights
    assert call(B=0, x=None, packed=None, q=None, g=None, out=None) == 0   # empty problem
    assert call(packed=None) == -1
    assert call(g=None) == -1
    assert call(x=ctypes.c_void_p(24)) == -3        # 16-byte alignment
    assert call(g=ctypes.c_void_p(40)) == -3


def test_mixer_projections_reject_invalid_arguments(lib):
    P = ctypes.c_void_p(16)
    S = None
    # in-projection: negative sizes, bad dtype, fp32 unsupported, empty, nulls, alignment
    assert lib.gtr_mixer_in_proj(P, P, P, P, P, P, -1, 4, 384, 6, 64, 64, 1, S) == -1
    assert lib.gtr_mixer_in_proj(P, P, P, P, P, P, 1, 4, 384, 6, 64, 64, 3, S) == -1
    assert lib.gtr_mixer_in_proj(P, P, P, P, P, P, 1, 4, 384, 6, 64, 64, 0, S) == -2
    assert lib.gtr_mixer_in_proj(None, None, None, None, None, None, 0, 4, 384, 6, 64, 64, 1, S) == 0
    assert lib.gtr_mixer_in_proj(P, None, P, P, P, P, 1, 4, 384, 6, 64, 64, 1, S) == -1
    assert lib.gtr_mixer_in_proj(ctypes.c_void_p(24), P, P, P, P, P, 1, 4, 384, 6, 64, 64, 1, S) == -3
    # out-projection
    assert lib.gtr_mixer_out_proj(P, P, P, -1, 384, 384, 1, S) == -1
    assert lib.gtr_mixer_out_proj(P, P, P, 4, 384, 384, 0, S) == -2
    assert lib.gtr_mixer_out_proj(None, None, None, 0, 384, 384, 1, S) == 0
    assert lib.gtr_mixer_out_proj(P, P, None, 4, 384, 384, 1, S) == -1
    assert lib.gtr_mixer_out_proj(P, ctypes.c_void_p(40), P, 4, 384, 384, 2, S) == -3


def test_sswiglu_rejects_invalid_arguments(lib):
    P = ctypes.c_void_p(16)
    S = None
    mix = lib.gtr_sswiglu_mix
    # u, conv_w, conv_b, h, B, gh, gw, C, ksize, dtype, stream
    assert mix(P, P, P, P, -1, 4, 4, 64, 3, 1, S) == -1             # negative size
    assert mix(P, P, P, P, 1, 4, 4, 64, 3, 5, S) == -1              # bad dtype
    assert mix(P, P, P, P, 1, 4, 4, 64, 4, 1, S) == -1              # even kernel
    assert mix(P, P, P, P, 1, 4, 4, 64, 0, 1, S) == -1
    assert mix(P, P, P, P, 1, 4, 4, 64, 5, 1, S) == -2              # only 3 x 3
    assert mix(P, P, P, P, 1, 4, 4, 64, 3, 0, S) == -2              # fp32
    assert mix(P, P, P, P, 1, 4, 4, 60, 3, 1, S) == -2              # C not a multiple of 8
    assert mix(None, None, None, None, 0, 4, 4, 64, 3, 1, S) == 0   # empty
    assert mix(None, None, None, None, 1, 4, 4, 0, 3, 2, S) == 0
    assert mix(P, None, P, P, 1, 4, 4, 64, 3, 1, S) == -1           # null weights
    assert mix(P, P, P, None, 1, 4, 4, 64, 3, 1, S) == -1
    assert mix(ctypes.c_void_p(24), P, None, P, 1, 4, 4, 64, 3, 1, S) == -3
    assert mix(P, P, ctypes.c_void_p(20), P, 1, 4, 4, 64, 3, 2, S) == -3
    # h overlapping u (u spans 1*4*4*128*2 = 4096 bytes from 4096): rejected before any launch
    U = ctypes.c_void_p(4096)
    assert mix(U, P, None, ctypes.c_void_p(4096 + 4080), 1, 4, 4, 64, 3, 1, S) == -1
    assert mix(U, P, None, ctypes.c_void_p(4096 - 2048 + 16), 1, 4, 4, 64, 3, 1, S) == -1
    assert mix(U, P, None, U, 1, 4, 4, 64, 3, 1, S) == -1
    fwd = lib.gtr_sswiglu_fwd
    # x, w_in, conv_w, conv_b, w_out, u, h, y, B, gh, gw, d_model, C, ksize, dtype, stream
    assert fwd(P, P, P, P, P, P, P, P, 1, 4, 4, -384, 1024, 3, 1, S) == -1
    assert fwd(P, P, P, P, P, P, P, P, 1, 4, 4, 384, 1024, 3, 0, S) == -2
    assert fwd(None, None, None, None, None, None, None, None, 1, 4, 4, 0, 1024, 3, 1, S) == 0
    assert fwd(P, P, P, P, P, P, None, P, 1, 4, 4, 384, 1024, 3, 1, S) == -1
    assert fwd(P, P, P, P, P, P, P, ctypes.c_void_p(8), 1, 4, 4, 384, 1024, 3, 1, S) == -3


def test_stack_rejects_invalid_arguments(lib):
    P = ctypes.c_void_p(16)
    S = None
    fwd = lib.gtr_stack_fwd
    blk = (binding.BlockWeights * 2)()
    for b in blk:
        for n in binding.BLOCK_FIELDS:
            setattr(b, n, 4096)
    need = lib.gtr_stack_workspace_bytes(1, 8, 8, 384, 6, 64, 64, 1024)
    assert need > 0 and lib.gtr_stack_workspace_bytes(-1, 8, 8, 384, 6, 64, 64, 1024) == 0
    W = ctypes.c_void_p(1 << 20)
    # x, blocks, nblocks, dirs, B, gh, gw, d_model, H, dk, dv, hidden, tau, chunk, dtype, ws, ws_bytes, stream
    args = [P, blk, 2, None, 1, 8, 8, 384, 6, 64, 64, 1024, 16.0, 64, 1, W, need, S]

    def call(**kw):
        a = list(args)
        names = ["x", "blocks", "n", "dirs", "B", "gh", "gw", "dm", "H", "dk", "dv", "hidden", "tau", "chunk",
                 "dtype", "ws", "ws_bytes", "stream"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return fwd(*a)

    assert call(B=-1) == -1
    assert call(n=-1) == -1
    assert call(tau=0.0) == -1
    assert call(dtype=0) == -2                     # fp32 activations
    assert call(dtype=7) == -1
    assert call(dk=48, dv=48, H=8) == -2           # no GLA kernel for dk = 48
    assert call(dm=320 + 8) == -2                  # the packed gate takes multiples of 64
    assert call(hidden=1020) == -2                 # S-SwiGLU width not a multiple of 8
    assert call(chunk=48) == -2
    assert call(n=0) == 0 and call(B=0) == 0       # empty: nothing launched
    assert call(x=None) == -1 and call(blocks=None) == -1 and call(ws=None) == -1
    assert call(ws_bytes=need - 1) == -4
    assert call(x=ctypes.c_void_p(20)) == -3
    blk[1].w_o = None
    assert call() == -1
    blk[1].w_o = 4096
    blk[0].conv_w = 4100
    assert call() == -3
    blk[0].conv_w = 4096
    bad_dirs = (ctypes.c_int * 2)(0, 4)            # per-batch rotation is not a block direction
    assert call(dirs=bad_dirs) == -1

"""The projections' tcgen05 GEMM across its kernels and tile shapes, against
the fp64 oracle.

gtr_mixer_out_proj is a plain C = A B.  The cases cover the single-CTA kernel
on 128 x 256 tiles (N a multiple of 256) and on 128 x 128 tiles (other N), the
CTA-pair kernel on 256 x 256 tiles (N a multiple of 256 and K >= 1024), ragged
M, N and K (rows, columns and K blocks past the edges are zero on load and
clipped on store), one-row problems, depths that are not a multiple of the
64-deep K block, and the four-output form of gtr_mixer_in_proj whose column
blocks are not multiples of the tile width.  Results are compared element by
element with the fp64 product rounded to the storage dtype (tests/parity.py);
at 16384 rows, on every 97th row.
"""
import pytest
import torch

import oracle
from linear_vision_backbone_b200 import binding, build
from tests.parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    build.build()
    binding.load()


def _pair(M, K, N, dtype, seed):
    gen = torch.Generator().manual_seed(seed)
    a = torch.randn(1, M, K, generator=gen).to(dtype)
    w = (torch.randn(K, N, generator=gen) / K ** 0.5).to(dtype)
    return a, w


@pytest.mark.parametrize("dtype", (torch.float16, torch.bfloat16))
@pytest.mark.parametrize("M,K,N", [
    (512, 384, 512),      # whole 256 x 256 pair tiles
    (300, 384, 768),      # ragged M: the second CTA of the last pair has 44 rows
    (1, 64, 256),         # one row
    (257, 136, 256),      # K not a multiple of 64, one row into a second pair tile
    (384, 1024, 384),     # 256 x 128 pair tiles (N = 384)
    (200, 96, 200),       # ragged N on 256 x 128 tiles
    (130, 384, 72),       # N narrower than one store box
    (512, 1024, 512),     # CTA pairs: whole 256 x 256 tiles
    (300, 1032, 768),     # CTA pairs: ragged M, K not a multiple of 64
    (1, 1024, 256),       # CTA pairs: one row (the second CTA's rows all past the edge)
])
def test_gemm_shapes(dtype, M, K, N):
    a, w = _pair(M, K, N, dtype, M + K + N)
    out = binding.mixer_out_proj(a.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert out.shape == (1, M, N)
    assert_close(out, oracle.linear(a, w), dtype, f"gemm {M}x{K}x{N}")


@pytest.mark.parametrize("dtype", (torch.float16, torch.bfloat16))
@pytest.mark.parametrize("K,N", [(384, 1536), (384, 2048), (1024, 384), (1024, 2048)])
def test_gemm_full_size_rows(dtype, K, N):
    # the 16k workload's projection shapes; every 97th row against the oracle
    M = 16384
    a, w = _pair(M, K, N, dtype, K + N)
    out = binding.mixer_out_proj(a.cuda(), w.cuda()).cpu()
    rows = torch.arange(0, M, 97)
    assert_close(out[:, rows], oracle.linear(a[:, rows], w), dtype, f"gemm 16384x{K}x{N} rows")


@pytest.mark.parametrize("H,dk", [(6, 64), (5, 64), (3, 32)])
def test_in_projection_four_outputs(H, dk):
    # column blocks of 384 (one and a half 256-wide tiles), 320 and 96 columns
    dtype, B, T, dm = torch.float16, 1, 1000, 384
    gen = torch.Generator().manual_seed(H * dk)
    x = torch.randn(B, T, dm, generator=gen).to(dtype)
    w = (torch.randn(dm, 4 * H * dk, generator=gen) / dm ** 0.5).to(dtype)
    outs = binding.mixer_in_proj(x.cuda(), w.cuda(), H, dk)
    torch.cuda.synchronize()
    ref = oracle.linear(x, w)
    for i, t in enumerate(outs):
        assert_close(t, ref[..., i * H * dk:(i + 1) * H * dk].reshape(B, T, H, dk), dtype, f"block {i}")
    rc, bits, _ = binding.device_status()
    assert rc == 0 and bits == 0, (rc, bits)

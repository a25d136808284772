"""Pins of the oracle's GTR block stack (oracle.gtr_block / gtr_stack / rmsnorm).

The stack is checked against a second fp64 implementation written here with
other formulas and other library routines: the GLA in its quadratic masked
form (no recurrence), the scan orders as index permutations built with torch,
torch's own rms_norm, logsigmoid and grouped conv2d.  Plus properties the
stack must have whatever its weights: the residual path alone is the identity,
one active block in a stack acts as that block alone with the direction its
index gives (LR, RL, TB, BT cycling, GTR article 方法详解 §1), and the stack on
the transposed grid with the vertical and horizontal orders exchanged is the
transposed stack.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from linear_vision_backbone_b200 import inputs

DIRS = ("LR", "RL", "TB", "BT")


# ---------------------------------------------------------------------------
# the second implementation (torch, fp64)

def _order(direction, gh, gw):
    """Grid index of every scan position, from an index grid."""
    grid = torch.arange(gh * gw).reshape(gh, gw)
    if direction in ("TB", "BT"):
        grid = grid.t()
    order = grid.reshape(-1)
    return order.flip(0) if direction in ("RL", "BT") else order


def _gla_quadratic(q, k, v, g, z, w, gh, gw, direction):
    """y = RMSNorm(o) * w * SiLU(z), o_t = sum_{s<=t} ((q_t * exp(G_t - G_s)) . k_s) v_s,
    G the running sum of g along the scan (the closed form of the recurrence)."""
    B, T, H, dk = q.shape
    idx = _order(direction, gh, gw)
    qs, ks, vs, gs = q[:, idx], k[:, idx], v[:, idx], g[:, idx]
    G = torch.cumsum(gs, dim=1)                                          # [B, T, H, dk]
    decay = torch.exp(G[:, :, None] - G[:, None, :])                     # [B, t, s, H, dk]
    A = torch.einsum("bthi,bshi,btshi->bhts", qs, ks, torch.tril(torch.ones(T, T, dtype=q.dtype))[None, :, :, None, None] * decay)
    o = torch.einsum("bhts,bshj->bthj", A, vs)
    y = F.rms_norm(o, (o.shape[-1],), weight=w, eps=1e-5) * F.silu(z[:, idx])
    out = torch.empty_like(y)
    out[:, idx] = y
    return out


def _block_torch(x, p, gh, gw, H, direction, tau=16.0, act=None):
    t = lambda a: None if a is None else torch.as_tensor(a).double()
    rnd = (lambda a: a) if act is None else (lambda a: a.to(act).double())
    r32 = (lambda a: a) if act is None else (lambda a: a.float().double())
    B, T, dm = x.shape
    n_q = p["w_up"].shape[1]
    dk = n_q // H
    dv = (p["w_in"].shape[1] - 2 * n_q) // (2 * H)
    a = rnd(F.rms_norm(x, (dm,), weight=t(p["norm_mixer"]), eps=1e-5))
    qkvz = rnd(a @ t(p["w_in"]))
    q, k, v, z = torch.split(qkvz, [n_q, n_q, H * dv, H * dv], dim=-1)
    u = a @ t(p["w_down"]) @ t(p["w_up"])
    if p.get("gate_bias") is not None:
        u = u + t(p["gate_bias"])
    g = r32(F.logsigmoid(u) / tau)
    y = rnd(_gla_quadratic(q.reshape(B, T, H, dk), k.reshape(B, T, H, dk), v.reshape(B, T, H, dv),
                           g.reshape(B, T, H, dk), z.reshape(B, T, H, dv), t(p.get("gla_norm")), gh, gw,
                           direction))
    x = r32(x + rnd(y.reshape(B, T, H * dv) @ t(p["w_o"])))
    c = rnd(F.rms_norm(x, (dm,), weight=t(p["norm_ffn"]), eps=1e-5))
    e = rnd(c @ t(p["w_e"]))
    C = e.shape[-1] // 2
    val = e[..., C:].reshape(B, gh, gw, C).permute(0, 3, 1, 2)
    taps = t(p["conv_w"]).permute(2, 0, 1)[:, None]                      # [C, 1, 3, 3]
    mixed = F.conv2d(val, taps, bias=t(p.get("conv_b")), padding=1, groups=C)
    h = rnd(F.silu(e[..., :C]) * mixed.permute(0, 2, 3, 1).reshape(B, T, C))
    return r32(x + rnd(h @ t(p["w_p"])))


def _stack_torch(x, blocks, gh, gw, H, dirs=None, act=None):
    x = torch.as_tensor(x).double()
    if act is not None:
        x = x.float().double()
    for i, p in enumerate(blocks):
        x = _block_torch(x, p, gh, gw, H, DIRS[i % 4] if dirs is None else dirs[i], act=act)
    return x.numpy()


def _small(nblocks, seed, **kw):
    kw = dict(dict(d_model=24, H=2, dk=8, dv=4, hidden=12, random_norms=True, bias_std=0.5), **kw)
    return inputs.make_stack(nblocks, 2, 5, 7, seed=seed, **kw)


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


# ---------------------------------------------------------------------------

def test_rmsnorm_closed_forms():
    x = np.array([[3.0, 4.0], [1.0, -1.0]])
    r = oracle.rmsnorm(x, eps=0.0)
    np.testing.assert_allclose(np.mean(r * r, axis=-1), 1.0, rtol=1e-15)
    np.testing.assert_allclose(r[0], [3 / np.sqrt(12.5), 4 / np.sqrt(12.5)], rtol=1e-15)
    # the weight scales each channel; epsilon shrinks the norm to m / (m + eps)
    np.testing.assert_allclose(oracle.rmsnorm(x, [2.0, -1.0], eps=0.0), r * [2.0, -1.0], rtol=1e-15)
    ms = np.mean(oracle.rmsnorm(x, eps=0.5) ** 2, axis=-1)
    np.testing.assert_allclose(ms, [12.5 / 13.0, 1.0 / 1.5], rtol=1e-14)


@pytest.mark.parametrize("nblocks", [1, 5])
def test_stack_matches_a_second_fp64_implementation(nblocks):
    # five blocks run LR, RL, TB, BT and LR again; dk != dv catches a wrong q|k|v|z split
    x, blocks = _small(nblocks, seed=40 + nblocks)
    got = oracle.gtr_stack(x, blocks, gh=5, gw=7, H=2)
    want = _stack_torch(x, blocks, 5, 7, 2)
    assert _rel(got, want) < 1e-12


@pytest.mark.parametrize("direction", DIRS)
def test_block_in_each_direction(direction):
    x, blocks = _small(1, seed=50)
    got = oracle.gtr_block(x, blocks[0], gh=5, gw=7, H=2, direction=direction)
    want = _stack_torch(x, blocks, 5, 7, 2, dirs=(direction,))
    assert _rel(got, want) < 1e-12


@pytest.mark.parametrize("act", [torch.float16, torch.bfloat16])
def test_stored_activations_match_the_second_implementation(act):
    # the storage roundings at each stage boundary, done by torch casts there
    x, blocks = _small(4, seed=60)
    got = oracle.gtr_stack(x, blocks, gh=5, gw=7, H=2, act_dtype=act)
    want = _stack_torch(x, blocks, 5, 7, 2, act=act)
    assert _rel(got, want) < 1e-12
    exact = oracle.gtr_stack(x, blocks, gh=5, gw=7, H=2)
    assert 1e-5 < _rel(got, exact) < 5e-2        # rounding happened, and stayed small


def test_residual_path_alone_is_the_identity():
    x, blocks = _small(6, seed=70)
    for p in blocks:
        p["w_o"] = torch.zeros_like(p["w_o"])
        p["w_p"] = torch.zeros_like(p["w_p"])
    got = oracle.gtr_stack(x, blocks, gh=5, gw=7, H=2)
    assert np.array_equal(got, x.double().numpy())


@pytest.mark.parametrize("j", range(4))
def test_one_active_block_takes_the_direction_of_its_index(j):
    x, blocks = _small(4, seed=80 + j)
    for i, p in enumerate(blocks):
        if i != j:
            p["w_o"] = torch.zeros_like(p["w_o"])
            p["w_p"] = torch.zeros_like(p["w_p"])
    got = oracle.gtr_stack(x, blocks, gh=5, gw=7, H=2)
    alone = oracle.gtr_block(x, blocks[j], gh=5, gw=7, H=2, direction=DIRS[j])
    assert _rel(got, alone) < 1e-14
    others = [oracle.gtr_block(x, blocks[j], gh=5, gw=7, H=2, direction=d) for d in DIRS if d != DIRS[j]]
    assert all(_rel(o, alone) > 1e-3 for o in others)


def test_transposed_grid_exchanges_the_orders():
    # LR/RL on a grid are TB/BT on its transpose; the 3x3 taps transpose with it
    gh, gw = 5, 7
    x, blocks = _small(4, seed=90)
    xt = x.reshape(2, gh, gw, -1).transpose(1, 2).reshape(2, gh * gw, -1)
    bt = []
    for p in blocks:
        q = dict(p)
        q["conv_w"] = p["conv_w"].transpose(0, 1).contiguous()
        bt.append(q)
    got = oracle.gtr_stack(x, blocks, gh=gh, gw=gw, H=2)
    swapped = oracle.gtr_stack(xt, bt, gh=gw, gw=gh, H=2, directions=("TB", "BT", "LR", "RL"))
    back = swapped.reshape(2, gw, gh, -1).transpose(0, 2, 1, 3).reshape(2, gh * gw, -1)
    assert _rel(back, got) < 1e-13


def test_a_planted_slip_is_caught(monkeypatch):
    # post-normalisation in place of pre-normalisation fails the comparison
    x, blocks = _small(2, seed=100)
    want = _stack_torch(x, blocks, 5, 7, 2)
    real = oracle.gtr_block

    def post_norm(x, p, **kw):
        return oracle.rmsnorm(real(x, p, **kw), p["norm_ffn"])

    monkeypatch.setattr(oracle, "gtr_block", post_norm)
    assert _rel(oracle.gtr_stack(x, blocks, gh=5, gw=7, H=2), want) > 1e-2

"""Pins of the fp64 oracle against results fixed independently of it.

Each test derives its expectation from something other than the oracle's own
recurrence: a different closed form of the same operator (the quadratic masked
form), a textbook special case (causal linear attention when every gate is 0;
the memoryless limit when every gate is -inf; T = 1), explicit grid flips and
transposes for the scan orders, exact special values of SiLU and logsigmoid,
and the torch implementation of logsigmoid for the gate.  The operator itself
is the Key-only gated recurrence of the GTR article (shuwu5.cn/article/3124),
方法详解 §1; the chunk states follow 方法详解 §4.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_vision_backbone_b200 import inputs


def _rand(seed, *shape, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _logsig(u):
    return np.minimum(u, 0.0) - np.log1p(np.exp(-np.abs(u)))


def _grid_case(seed, B=2, H=2, gh=3, gw=5, dk=4, dv=3, gate_scale=0.5):
    T = gh * gw
    q = _rand(seed, B, T, H, dk)
    k = _rand(seed + 1, B, T, H, dk)
    v = _rand(seed + 2, B, T, H, dv)
    g = _logsig(_rand(seed + 3, B, T, H, dk)) * gate_scale
    z = _rand(seed + 4, B, T, H, dv)
    return q, k, v, g, z


def _quadratic_o(q, k, v, g):
    """o_t = sum_{s<=t} sum_i q_t,i exp(Gam_t,i - Gam_s,i) k_s,i v_s, Gam = inclusive cumsum.

    The parallel (masked) form of the key-side gated recurrence, in raster (LR)
    order: the product of diag(exp g) from s+1 to t is exp(Gam_t - Gam_s).
    """
    B, T, H, dk = q.shape
    gam = np.cumsum(g, axis=1)
    o = np.zeros(v.shape)
    for t in range(T):
        dec = np.exp(gam[:, t:t + 1] - gam[:, : t + 1])            # [B, t+1, H, dk]
        sc = np.einsum("bhi,bshi,bshi->bsh", q[:, t], dec, k[:, : t + 1])
        o[:, t] = np.einsum("bsh,bshj->bhj", sc, v[:, : t + 1])
    return o


def test_quadratic_form_pins_recurrence():
    q, k, v, g, z = _grid_case(10)
    _, o = oracle.gla_fwd(q, k, v, g, z, gh=3, gw=5, direction="LR", return_o=True)
    ref = _quadratic_o(q, k, v, g)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


def test_zero_gate_is_causal_linear_attention():
    q, k, v, g, z = _grid_case(20, gh=4, gw=4)
    g = np.zeros_like(g)
    _, o = oracle.gla_fwd(q, k, v, g, z, gh=4, gw=4, direction="LR", return_o=True)
    # textbook causal linear attention: (tril(Q K^T)) V per (batch, head)
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            Q, K, V = q[b, :, h], k[b, :, h], v[b, :, h]
            ref = np.tril(Q @ K.T) @ V
            np.testing.assert_allclose(o[b, :, h], ref, rtol=1e-12, atol=1e-12)


def test_minus_infinite_gate_is_memoryless():
    q, k, v, g, z = _grid_case(30)
    g = np.full_like(g, -1e4)          # exp(-1e4) == 0.0 exactly in fp64
    _, o = oracle.gla_fwd(q, k, v, g, z, gh=3, gw=5, direction="LR", return_o=True)
    ref = np.einsum("bthi,bthi->bth", q, k)[..., None] * v
    np.testing.assert_allclose(o, ref, rtol=1e-13, atol=1e-13)


def test_single_token():
    q, k, v, g, z = _grid_case(40, gh=1, gw=1)
    _, o = oracle.gla_fwd(q, k, v, g, z, gh=1, gw=1, direction="TB", return_o=True)
    ref = np.einsum("bthi,bthi->bth", q, k)[..., None] * v
    np.testing.assert_allclose(o, ref, rtol=1e-14, atol=1e-14)


def test_hand_worked_two_token_example():
    # dk = dv = 1 over a 1x2 grid (LR), alpha = exp(g) = 1/2 at the second token:
    #   S_0 = k0 v0 = 2*3 = 6,            o_0 = q0 S_0 = 1*6 = 6
    #   S_1 = 1/2 * 6 + k1 v1 = 3 + (-1)*4 = -1,   o_1 = q1 S_1 = 5*(-1) = -5
    q = np.array([1.0, 5.0]).reshape(1, 2, 1, 1)
    k = np.array([2.0, -1.0]).reshape(1, 2, 1, 1)
    v = np.array([3.0, 4.0]).reshape(1, 2, 1, 1)
    g = np.array([math.log(0.25), -math.log(2.0)]).reshape(1, 2, 1, 1)
    z = np.zeros((1, 2, 1, 1))
    y, o = oracle.gla_fwd(q, k, v, g, z, gh=1, gw=2, direction="LR", return_o=True)
    assert o.ravel().tolist() == [6.0, -5.0]
    assert y.ravel().tolist() == [0.0, 0.0]            # SiLU(0) = 0


def _flipT(a):
    return a[:, ::-1]


def _transpose_grid(a, gh, gw):
    B, T, H, d = a.shape
    return a.reshape(B, gh, gw, H, d).transpose(0, 2, 1, 3, 4).reshape(B, T, H, d)


@pytest.mark.parametrize("gh,gw", [(3, 5), (4, 4), (1, 6), (7, 2)])
def test_scan_orders_against_grid_flips_and_transposes(gh, gw):
    q, k, v, g, z = _grid_case(50, gh=gh, gw=gw)
    args = (q, k, v, g, z)
    lr = oracle.gla_fwd(*args, gh=gh, gw=gw, direction="LR")
    rl = oracle.gla_fwd(*args, gh=gh, gw=gw, direction="RL")
    tb = oracle.gla_fwd(*args, gh=gh, gw=gw, direction="TB")
    bt = oracle.gla_fwd(*args, gh=gh, gw=gw, direction="BT")
    # RL = LR on the reversed token sequence, reversed back
    ref_rl = _flipT(oracle.gla_fwd(*[_flipT(a) for a in args], gh=gh, gw=gw, direction="LR"))
    # TB = LR on the transposed grid (gw x gh), transposed back
    ta = [_transpose_grid(a, gh, gw) for a in args]
    ref_tb = _transpose_grid(oracle.gla_fwd(*ta, gh=gw, gw=gh, direction="LR"), gw, gh)
    # BT = TB reversed = LR on the reversed transposed grid
    ref_bt = _transpose_grid(_flipT(oracle.gla_fwd(*[_flipT(a) for a in ta], gh=gw, gw=gh,
                                                   direction="LR")), gw, gh)
    np.testing.assert_allclose(rl, ref_rl, rtol=0, atol=0)
    np.testing.assert_allclose(tb, ref_tb, rtol=0, atol=0)
    np.testing.assert_allclose(bt, ref_bt, rtol=0, atol=0)
    assert not np.allclose(lr, rl)
    if gh > 1 and gw > 1:          # on a single row or column TB visits tokens as LR does
        assert not np.allclose(lr, tb)
    else:
        np.testing.assert_array_equal(lr, tb)


@pytest.mark.parametrize("gh,gw", [(3, 5), (4, 4), (2, 7)])
def test_scan_index_maps(gh, gw):
    T = gh * gw
    grid = np.arange(T).reshape(gh, gw)
    expect = {
        "LR": grid.ravel(),
        "RL": grid.ravel()[::-1],
        "TB": grid.T.ravel(),
        "BT": grid.T.ravel()[::-1],
    }
    for d, seq in expect.items():
        got = [oracle.scan_index(d, s, gh, gw) for s in range(T)]
        assert got == seq.tolist(), d


def test_rotate_batch_uses_b_mod_4():
    q, k, v, g, z = _grid_case(60, B=6, gh=3, gw=4)
    rot = oracle.gla_fwd(q, k, v, g, z, gh=3, gw=4, direction="ROTATE")
    names = ["LR", "RL", "TB", "BT"]
    for b in range(6):
        one = oracle.gla_fwd(*(a[b:b + 1] for a in (q, k, v, g, z)), gh=3, gw=4,
                             direction=names[b % 4])
        np.testing.assert_array_equal(rot[b:b + 1], one)


def test_rmsnorm_and_silu_closed_forms():
    q, k, v, g, z = _grid_case(70, dv=5)
    # eps = 0: every normalised row has mean square exactly 1 (up to rounding)
    ones = np.zeros_like(z) + math.log(3.0)      # sigmoid(ln 3) = 3/4 exactly
    y, o = oracle.gla_fwd(q, k, v, g, ones, gh=3, gw=5, eps=0.0, return_o=True)
    n = y / (0.75 * math.log(3.0))
    np.testing.assert_allclose(np.mean(n ** 2, axis=-1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(n * np.sqrt(np.mean(o ** 2, axis=-1, keepdims=True)), o,
                               rtol=1e-12, atol=1e-12)
    # eps > 0: mean square m/(m+eps)
    eps = 0.37
    y2, o2 = oracle.gla_fwd(q, k, v, g, ones, gh=3, gw=5, eps=eps, return_o=True)
    m = np.mean(o2 ** 2, axis=-1)
    np.testing.assert_allclose(np.mean((y2 / (0.75 * math.log(3.0))) ** 2, axis=-1),
                               m / (m + eps), rtol=1e-12)
    # the weight multiplies each output channel
    w = np.array([2.0, -1.0, 0.5, 0.0, 3.0])
    y3 = oracle.gla_fwd(q, k, v, g, ones, w, gh=3, gw=5, eps=eps)
    np.testing.assert_allclose(y3, y2 * w, rtol=1e-14, atol=1e-15)
    # SiLU(0) = 0; SiLU(-inf) -> 0; SiLU(z) ~ z for large z
    y0 = oracle.gla_fwd(q, k, v, g, np.zeros_like(z), gh=3, gw=5)
    assert np.all(y0 == 0.0)
    big = np.full_like(z, 60.0)
    yb = oracle.gla_fwd(q, k, v, g, big, gh=3, gw=5, eps=eps)
    np.testing.assert_allclose(yb / 60.0, y2 / (0.75 * math.log(3.0)), rtol=1e-12)


def test_gate_against_torch_logsigmoid_and_special_values():
    gen = torch.Generator().manual_seed(5)
    x = torch.randn(3, 7, 24, generator=gen, dtype=torch.float64)
    wd = torch.randn(24, 4, generator=gen, dtype=torch.float64) / math.sqrt(24)
    wu = torch.randn(4, 10, generator=gen, dtype=torch.float64) / 2
    b = torch.randn(10, generator=gen, dtype=torch.float64)
    got = oracle.gate(x, wd, wu, b, tau=16.0)
    ref = torch.nn.functional.logsigmoid(x @ wd @ wu + b) / 16.0
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-13, atol=1e-15)
    assert np.all(got <= 0.0)
    # u = 0 -> -ln 2 / tau;  u = ln 3 -> ln(3/4) / tau;  u = -800 -> -800 / tau
    xz = np.zeros((1, 24))
    for bias, expect in [(0.0, -math.log(2.0)), (math.log(3.0), math.log(0.75)), (-800.0, -800.0)]:
        gg = oracle.gate(xz, wd, wu, np.full(10, bias), tau=4.0)
        np.testing.assert_allclose(gg, expect / 4.0, rtol=1e-15)
    # bias=None equals an all-zero bias
    np.testing.assert_array_equal(oracle.gate(x, wd, wu, None), oracle.gate(x, wd, wu, np.zeros(10)))


@pytest.mark.parametrize("chunk", [1, 2, 4, 5, 16])
def test_chunk_states_against_explicit_sum(chunk):
    q, k, v, g, z = _grid_case(80, gh=3, gw=5)
    st = oracle.chunk_states(k, v, g, gh=3, gw=5, direction="LR", chunk=chunk)
    T = 15
    gam = np.cumsum(g, axis=1)
    nc = (T + chunk - 1) // chunk
    assert st.shape[2] == nc
    for c in range(nc):
        e = min((c + 1) * chunk, T) - 1
        dec = np.exp(gam[:, e:e + 1] - gam[:, : e + 1])            # [B, s, H, dk]
        ref = np.einsum("bshi,bshj->bhij", dec * k[:, : e + 1], v[:, : e + 1])
        np.testing.assert_allclose(st[:, :, c], ref, rtol=1e-12, atol=1e-12)


def _chunkwise_midpoint(q, k, v, g, C):
    """The chunkwise decomposition the CUDA path computes, written out in fp64.

    Within chunk c (local positions j), G_j = inclusive cumsum of g, Gm = G at
    the chunk's middle position, Gam = G at its last position:
      o_j = (q_j * e^{G_j - Gm}) . (e^{Gm} * S_prev)                 inter-chunk
          + sum_{i<=j} [(q_j * e^{G_j - Gm}) . (k_i * e^{Gm - G_i})] v_i   intra
      S   = e^{Gam} * S_prev + sum_i (k_i * e^{Gam - G_i})^T v_i        state
    (GTR article, 方法详解 §4: block summaries, boundary scan, block outputs.)
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S = np.zeros((B, H, dk, dv))
    for c0 in range(0, T, C):
        n = min(C, T - c0)
        G = np.cumsum(g[:, c0:c0 + n], axis=1)                     # [B, n, H, dk]
        Gm = G[:, (n - 1) // 2]
        Gam = G[:, n - 1]
        qt = q[:, c0:c0 + n] * np.exp(G - Gm[:, None])
        kt = k[:, c0:c0 + n] * np.exp(Gm[:, None] - G)
        kh = k[:, c0:c0 + n] * np.exp(Gam[:, None] - G)
        Sp = np.exp(Gm)[..., None] * S                              # [B, H, dk, dv]
        inter = np.einsum("bjhi,bhiv->bjhv", qt, Sp)
        P = np.einsum("bjhi,bshi->bhjs", qt, kt) * np.tril(np.ones((n, n)))
        intra = np.einsum("bhjs,bshv->bjhv", P, v[:, c0:c0 + n])
        o[:, c0:c0 + n] = inter + intra
        S = np.exp(Gam)[..., None] * S + np.einsum("bjhi,bjhv->bhiv", kh, v[:, c0:c0 + n])
    return o


@pytest.mark.parametrize("C", [1, 3, 4, 8, 16])
def test_chunkwise_decomposition_matches_oracle(C):
    q, k, v, g, z = _grid_case(90, gh=4, gw=5)
    _, o = oracle.gla_fwd(q, k, v, g, z, gh=4, gw=5, return_o=True)
    np.testing.assert_allclose(_chunkwise_midpoint(q, k, v, g, C), o, rtol=1e-11, atol=1e-11)


def test_planted_mistakes_are_caught():
    """Plausible slips in the recurrence each break one of the pins above."""
    q, k, v, g, z = _grid_case(100)
    quad = _quadratic_o(q, k, v, g)

    def recurrence(decay_value_side=False, decay_after_update=False, exclusive=False):
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        o = np.zeros((B, T, H, dv))
        S = np.zeros((B, H, dk, dv))
        for t in range(T):
            a = np.exp(g[:, t])                                     # [B, H, dk]
            kv = np.einsum("bhi,bhj->bhij", k[:, t], v[:, t])
            if exclusive:
                o[:, t] = np.einsum("bhi,bhij->bhj", q[:, t], S)
            if decay_value_side:
                S = S * a[:, :, None, :dv] + kv
            elif decay_after_update:
                S = a[..., None] * (S + kv)
            else:
                S = a[..., None] * S + kv
            if not exclusive:
                o[:, t] = np.einsum("bhi,bhij->bhj", q[:, t], S)
        return o

    np.testing.assert_allclose(recurrence(), quad, rtol=1e-12, atol=1e-12)
    for slip in ("decay_value_side", "decay_after_update", "exclusive"):
        assert not np.allclose(recurrence(**{slip: True}), quad, rtol=1e-6, atol=1e-6), slip


def test_inputs_are_deterministic_and_shaped():
    wl = inputs.WORKLOADS["640"]
    a = inputs.make_inputs(wl)
    b = inputs.make_inputs(wl)
    for key in a:
        assert torch.equal(a[key], b[key]), key
    assert a["q"].shape == (1, 1600, 6, 64) and a["q"].dtype == torch.float16
    assert a["x"].shape == (1, 1600, 384) and a["w_up"].shape == (16, 384)
    # q = x W with W ~ N(0, 1/384) comes out ~ N(0, 1)
    assert 0.9 < float(a["q"].float().std()) < 1.1
    t = inputs.make_inputs(inputs.WORKLOADS["tiny"])
    assert t["g"].dtype == torch.float32 and float(t["g"].max()) <= 0.0
    assert t["q"].dtype == torch.float32 and t["q"].shape == (1, 64, 1, 16)


def test_oracle_reproduces_its_stored_tiny_output():
    import json
    import os
    doc = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")))
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.make_inputs(wl)
    y = oracle.gla_fwd(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], gh=wl.gh, gw=wl.gw)
    stored = np.array([float.fromhex(v) for v in doc["y"]]).reshape(doc["shape"])
    np.testing.assert_allclose(y, stored, rtol=1e-13, atol=1e-15)


def test_linear_is_the_matrix_product():
    # the projections' oracle against the definition of the product, summed term by term
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 4, 5))
    w = rng.standard_normal((5, 7))
    got = oracle.linear(x, w)
    ref = np.zeros((3, 4, 7))
    for a in range(3):
        for b in range(4):
            for j in range(7):
                ref[a, b, j] = sum(x[a, b, i] * w[i, j] for i in range(5))
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)

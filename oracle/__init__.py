"""fp64 CPU oracle for the Key-only GLA token mixer of GTR.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library in
``linear_vision_backbone_b200`` never imports, links or runs it, and the two
share no code: the oracle is plain C (``gla_oracle.c``) compiled with gcc, in
IEEE fp64 (no fast-math), driven through ctypes from here.

Functions (each cites the page passage it follows in ``gla_oracle.c``):

* :func:`gate` -- ``g = logsigmoid(x W_down W_up + b) / tau`` (GTR article,
  方法详解 §1, low-rank forget gate with temperature).
* :func:`gla_fwd` -- the token-by-token recurrence ``S_t = diag(exp g_t) S_{t-1}
  + k_t^T v_t``, ``o_t = q_t S_t``, then ``RMSNorm(o_t) * SiLU(z_t)``, over the
  grid in one of the four scan orders, written back in grid order (GTR article,
  方法详解 §1).
* :func:`chunk_states` -- the state after every chunk of scan positions (GTR
  article, 方法详解 §4, the boundary states of the chunkwise operator).
* :func:`scan_index` -- the grid index visited at a scan position.
* :func:`linear` -- the token mixer's projections, a plain matrix product.
* :func:`dwconv2d`, :func:`sswiglu_mix`, :func:`sswiglu` -- the Spatial SwiGLU
  feed-forward block: SiLU(gate) times the depthwise-convolved value branch on
  the token grid, between two projections (GTR article, 方法详解 §2), in
  numpy fp64.
* :func:`rmsnorm`, :func:`gtr_block`, :func:`gtr_stack` -- blocks of the
  12-block backbone (GTR article, 方法详解 §1: the GLA at each block's core,
  scan directions cycling LR, RL, TB, BT with depth) with the S-SwiGLU half,
  pre-normalised and residual (the pages leave the wiring blank), in numpy
  fp64, optionally rounding what each stage hands on to a 16-bit storage type.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
results fixed independently of it (the quadratic masked form, plain causal
linear attention at g = 0, the memoryless limit, T = 1, explicit grid flips and
transposes, closed forms of the gate, scipy's 2-D correlation and brute-force
loops for the depthwise convolution); the block stack in
``tests/test_oracle_stack.py`` against a second fp64 implementation (the GLA's
quadratic masked form, torch's rms_norm and grouped conv2d) and against
properties of the stack (residual identity, direction by block index, grid
transposition).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gla_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

DIRS = {"LR": 0, "RL": 1, "TB": 2, "BT": 3, "ROTATE": 4}


def build(force: bool = False) -> str:
    """Compile ``gla_oracle.c`` with gcc (fp64, -O2, OpenMP, no fast-math)."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            i, l, d = ctypes.c_int, ctypes.c_long, ctypes.c_double
            lib.oracle_gate_f64.argtypes = [P, P, P, P, P, l, i, i, i, d]
            lib.oracle_gate_f64.restype = i
            lib.oracle_gla_fwd_f64.argtypes = [P, P, P, P, P, P, P, P, i, i, i, i, i, i, i, d]
            lib.oracle_gla_fwd_f64.restype = i
            lib.oracle_gla_chunk_states_f64.argtypes = [P, P, P, P, i, i, i, i, i, i, i, i]
            lib.oracle_gla_chunk_states_f64.restype = i
            lib.oracle_scan_index.argtypes = [i, l, l, l]
            lib.oracle_scan_index.restype = l
            lib.oracle_set_threads.argtypes = [i]
            lib.oracle_set_threads.restype = i
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    """Exact widening to a C-contiguous fp64 array (accepts numpy or torch CPU tensors)."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        a = a.double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> int:
    """Set the OpenMP thread count of the oracle; returns the count in effect."""
    return int(_load().oracle_set_threads(int(n)))


def scan_index(direction: str, s: int, gh: int, gw: int) -> int:
    return int(_load().oracle_scan_index(DIRS[direction], int(s), int(gh), int(gw)))


def gate(x, w_down, w_up, bias=None, tau: float = 16.0) -> np.ndarray:
    """g[n, :] = logsigmoid(x[n] @ w_down @ w_up + bias) / tau, fp64.

    ``x`` may have any leading shape; the last axis is the model width.
    """
    x = _f64(x)
    lead = x.shape[:-1]
    dm = x.shape[-1]
    x2 = x.reshape(-1, dm)
    wd, wu = _f64(w_down), _f64(w_up)
    rank, HD = wu.shape
    assert wd.shape == (dm, rank)
    b = None if bias is None else _f64(bias).reshape(HD)
    out = np.empty((x2.shape[0], HD), dtype=np.float64)
    rc = _load().oracle_gate_f64(_ptr(x2), _ptr(wd), _ptr(wu), None if b is None else _ptr(b),
                                 _ptr(out), x2.shape[0], dm, rank, HD, float(tau))
    if rc != 0:
        raise ValueError(f"oracle_gate_f64 rejected its arguments (rc={rc})")
    return out.reshape(*lead, HD)


def gla_fwd(q, k, v, g, z, w=None, *, gh: int, gw: int, direction: str = "LR",
            eps: float = 1e-5, return_o: bool = False):
    """y = RMSNorm(o) * SiLU(z) with o from the Key-only gated recurrence, fp64.

    q, k, g: [B, T, H, dk]; v, z: [B, T, H, dv]; w: [dv] or None; T = gh * gw.
    Returns y (and o before the normalisation when ``return_o``).
    """
    q, k, v, g, z = (_f64(a) for a in (q, k, v, g, z))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert T == gh * gw and k.shape == q.shape and g.shape == q.shape
    assert v.shape == (B, T, H, dv) and z.shape == v.shape
    wv = None if w is None else _f64(w).reshape(dv)
    y = np.empty((B, T, H, dv), dtype=np.float64)
    o = np.empty_like(y) if return_o else None
    rc = _load().oracle_gla_fwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(z),
                                    None if wv is None else _ptr(wv), _ptr(y),
                                    None if o is None else _ptr(o),
                                    B, H, gh, gw, dk, dv, DIRS[direction], float(eps))
    if rc != 0:
        raise ValueError(f"oracle_gla_fwd_f64 rejected its arguments (rc={rc})")
    return (y, o) if return_o else y


def linear(x, w) -> np.ndarray:
    """x W in fp64 (the token mixer's projections, GTR article 方法详解 §1):
    x [..., K], w [K, n] -> [..., n].  A plain matrix product."""
    x64, w64 = _f64(x), _f64(w)
    return np.matmul(x64, w64)


def chunk_states(k, v, g, *, gh: int, gw: int, direction: str = "LR", chunk: int = 64) -> np.ndarray:
    """State after each chunk of ``chunk`` scan positions: [B, H, ceil(T/chunk), dk, dv]."""
    k, v, g = (_f64(a) for a in (k, v, g))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    nc = (T + chunk - 1) // chunk
    st = np.empty((B, H, nc, dk, dv), dtype=np.float64)
    rc = _load().oracle_gla_chunk_states_f64(_ptr(k), _ptr(v), _ptr(g), _ptr(st), B, H, gh, gw,
                                             dk, dv, DIRS[direction], int(chunk))
    if rc != 0:
        raise ValueError(f"oracle_gla_chunk_states_f64 rejected its arguments (rc={rc})")
    return st


def silu(a) -> np.ndarray:
    """SiLU(a) = a * sigmoid(a) in fp64, written so that neither branch overflows."""
    a = _f64(a)
    e = np.exp(-np.abs(a))
    return np.where(a >= 0, a / (1.0 + e), a * e / (1.0 + e))


def dwconv2d(val, weight, bias=None, *, gh: int, gw: int) -> np.ndarray:
    """Depthwise 2-D cross-correlation of a channels-last token grid, fp64.

    val [B, gh*gw, C] (token t = row * gw + column), weight [k, k, C] (odd k),
    bias [C] or None -> [B, gh*gw, C] with
        out[b, y, x, c] = bias[c] + sum_{i,j} weight[i, j, c] * val[b, y+i-r, x+j-r, c],
    r = k // 2, and val = 0 outside the grid ("same" size, zero padding).  This
    is the local mixing of the S-SwiGLU value branch after it is laid out as the
    2-D token grid (GTR article, 方法详解 §2, Spatial SwiGLU).  Written as the k*k
    shifted copies of the zero-padded grid, summed tap by tap."""
    v = _f64(val)
    w = _f64(weight)
    B, T, C = v.shape
    k = w.shape[0]
    if T != gh * gw or w.shape != (k, k, C) or k % 2 != 1:
        raise ValueError("dwconv2d: shapes")
    r = k // 2
    grid = v.reshape(B, gh, gw, C)
    pad = np.zeros((B, gh + 2 * r, gw + 2 * r, C))
    pad[:, r:r + gh, r:r + gw] = grid
    out = np.zeros((B, gh, gw, C))
    for i in range(k):
        for j in range(k):
            out += w[i, j] * pad[:, i:i + gh, j:j + gw]
    if bias is not None:
        out += _f64(bias)
    return out.reshape(B, T, C)


def sswiglu_mix(u, weight, bias=None, *, gh: int, gw: int) -> np.ndarray:
    """The S-SwiGLU hidden activation from the expanded tokens, fp64 (GTR
    article, 方法详解 §2): u [B, T, 2C] holds the gate branch in its first C
    channels and the value branch in the last C; the value branch is mixed on
    the token grid by the depthwise convolution and multiplied by SiLU of the
    gate branch: h = SiLU(u_gate) * dwconv2d(u_value) -> [B, T, C]."""
    u = _f64(u)
    C = u.shape[-1] // 2
    return silu(u[..., :C]) * dwconv2d(u[..., C:], weight, bias, gh=gh, gw=gw)


def sswiglu(x, w_in, weight, bias, w_out, *, gh: int, gw: int) -> np.ndarray:
    """The S-SwiGLU feed-forward block in fp64 (GTR article, 方法详解 §2): the
    expansion x W_in -> [gate | value], the grid-mixed gated product h, and the
    projection back h W_out.  x [B, T, Cm], w_in [Cm, 2C], w_out [C, Cm]."""
    return linear(sswiglu_mix(linear(x, w_in), weight, bias, gh=gh, gw=gw), w_out)


# ---------------------------------------------------------------------------
# The stack of GTR blocks (GTR article, 方法详解 §1: a single-scale topology of
# 12 blocks, each built around the Key-only GLA, whose scan direction cycles
# LR, RL, TB, BT from Block 1 to Block 12; 方法详解 §2: the Spatial SwiGLU
# feed-forward half).  The pages do not print a block's wiring.  Reading used
# here: pre-normalisation with a residual around each half,
#     x <- x + W_o-projection of GLA(mixer inputs of RMSNorm(x) * gamma_mixer)
#     x <- x + S-SwiGLU(RMSNorm(x) * gamma_ffn),
# with RMSNorm's epsilon 1e-5 as for the GLA output, the gate computed from the
# same normalised input as q, k, v and z, and no final normalisation.

STACK_DIRS = ("LR", "RL", "TB", "BT")


def rmsnorm(x, weight=None, eps: float = 1e-5) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * weight over the last axis, fp64."""
    x = _f64(x)
    r = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return r if weight is None else r * _f64(weight)


def store(a, dtype):
    """``a`` rounded to the storage type ``dtype`` (a torch dtype, or None for
    no rounding) and widened back to fp64: the value a stage hands to the next
    when the pipeline keeps it in that type.  torch's CPU cast rounds fp64 to
    fp32 and then to a 16-bit type, each step to nearest-even: the rounding of
    a pipeline that computes in fp32 and stores 16 bits."""
    a = _f64(a)
    if dtype is None:
        return a
    import torch
    return torch.from_numpy(a).to(dtype).double().numpy()


def gtr_block(x, p, *, gh: int, gw: int, H: int, direction: str, tau: float = 16.0,
              act_dtype=None):
    """One GTR block on the fp64 residual stream x [B, T, d_model].

    ``p`` holds the block's weights: norm_mixer [d_model], w_in [d_model,
    2 H dk + 2 H dv] (column blocks W_q | W_k | W_v | W_z), w_down [d_model, r],
    w_up [r, H dk], gate_bias [H dk] or None, gla_norm [dv] or None, w_o [H dv,
    d_model], norm_ffn [d_model], w_e [d_model, 2C] (gate | value), conv_w
    [3, 3, C], conv_b [C] or None, w_p [C, d_model].

    ``act_dtype`` (None, torch.float16 or torch.bfloat16): when given, every
    tensor that one stage hands to the next is rounded to it as a pipeline that
    stores activations in that type does (the normalised inputs, q, k, v, z,
    the GLA output, the S-SwiGLU expansion and hidden activation, and both
    projections' outputs), the gate's g and the residual stream to fp32; each
    stage computes in fp64 from the rounded values it receives.
    """
    f32 = None if act_dtype is None else __import__("torch").float32
    s = lambda a: store(a, act_dtype)
    x = _f64(x)
    B, T, dm = x.shape
    w_in = _f64(p["w_in"])
    n_q = _f64(p["w_up"]).shape[1]
    dk = n_q // H
    dv = (w_in.shape[1] - 2 * n_q) // (2 * H)
    a = s(rmsnorm(x, p["norm_mixer"]))
    qkvz = s(linear(a, w_in))
    q = qkvz[..., :n_q].reshape(B, T, H, dk)
    k = qkvz[..., n_q:2 * n_q].reshape(B, T, H, dk)
    v = qkvz[..., 2 * n_q:2 * n_q + H * dv].reshape(B, T, H, dv)
    z = qkvz[..., 2 * n_q + H * dv:].reshape(B, T, H, dv)
    g = store(gate(a, p["w_down"], p["w_up"], p.get("gate_bias"), tau), f32).reshape(B, T, H, dk)
    y = s(gla_fwd(q, k, v, g, z, p.get("gla_norm"), gh=gh, gw=gw, direction=direction))
    x = store(x + s(linear(y.reshape(B, T, H * dv), p["w_o"])), f32)
    c = s(rmsnorm(x, p["norm_ffn"]))
    u = s(linear(c, p["w_e"]))
    h = s(sswiglu_mix(u, p["conv_w"], p.get("conv_b"), gh=gh, gw=gw))
    return store(x + s(linear(h, p["w_p"])), f32)


def gtr_stack(x, blocks, *, gh: int, gw: int, H: int, tau: float = 16.0, directions=None,
              act_dtype=None) -> np.ndarray:
    """The blocks applied in order to x [B, T, d_model]; block i scans in
    direction ``directions[i]``, by default STACK_DIRS[i % 4] (LR, RL, TB, BT,
    LR, ...).  Returns the residual stream after the last block, fp64."""
    x = _f64(x)
    if act_dtype is not None:
        x = store(x, __import__("torch").float32)
    for i, p in enumerate(blocks):
        d = STACK_DIRS[i % 4] if directions is None else directions[i]
        x = gtr_block(x, p, gh=gh, gw=gw, H=H, direction=d, tau=tau, act_dtype=act_dtype)
    return x

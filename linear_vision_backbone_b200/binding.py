"""Thin ctypes binding of ``include/gtr_gla.h`` (argument marshalling only).

Every step of the operator runs inside ``_build/libgtr_gla.so``; this module
only checks torch tensors, passes their device pointers and the current CUDA
stream through the C ABI, and turns status codes into exceptions.  There is no
Python or CPU fallback: if the library is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_build", "libgtr_gla.so")

DTYPE_IDS = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
DIR_IDS = {"LR": 0, "RL": 1, "TB": 2, "BT": 3, "ROTATE": 4}
PATH_IDS = {"auto": 0, "simt": 1, "tc": 2}
PATH_NAMES = {1: "simt", 2: "tc"}

EXPORTS = (
    "gtr_abi_version", "gtr_status_string", "gtr_gate_fwd", "gtr_gla_fwd", "gtr_gla_fwd_timed",
    "gtr_gla_chunk_states", "gtr_gla_workspace_bytes", "gtr_gla_set_workspace",
    "gtr_gla_set_path", "gtr_gla_path_for", "gtr_last_device_status", "gtr_gla_segment_chunks",
    "gtr_gla_fwd_noalloc", "gtr_gate_packed_bytes", "gtr_gate_pack", "gtr_gate_fwd_packed",
    "gtr_gla_segment_count", "gtr_gla_fwd_gated", "gtr_gla_fwd_gated_timed", "gtr_mixer_in_proj",
    "gtr_mixer_out_proj", "gtr_sswiglu_mix", "gtr_sswiglu_fwd", "gtr_stack_workspace_bytes",
    "gtr_stack_fwd",
)

BLOCK_FIELDS = ("norm_mixer", "w_in", "gate_packed", "gate_bias", "gla_norm", "w_o", "norm_ffn", "w_e",
                "conv_w", "conv_b", "w_p")


class BlockWeights(ctypes.Structure):
    """``gtr_block_weights``: one block's device pointers, in the header's order."""
    _fields_ = [(n, ctypes.c_void_p) for n in BLOCK_FIELDS]

_lock = threading.Lock()
_lib = None


class GtrError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {msg} (status {status})")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"CUDA library {path} is missing; build it with "
                "`python -m linear_vision_backbone_b200.build` (there is no fallback)")
        lib = ctypes.CDLL(path)
        P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        sig = {
            "gtr_abi_version": ([], I),
            "gtr_status_string": ([I], ctypes.c_char_p),
            "gtr_gate_fwd": ([P, I, P, P, P, P, I, I, I, I, I, I, F, P], I),
            "gtr_gla_fwd": ([P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P], I),
            "gtr_gla_fwd_timed": ([P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, P], I),
            "gtr_gla_chunk_states": ([P, P, P, P, I, I, I, I, I, I, I, I, I, P], I),
            "gtr_gla_workspace_bytes": ([I, I, I, I, I, I, I, I], Z),
            "gtr_gla_set_workspace": ([P, Z], I),
            "gtr_gla_set_path": ([I], I),
            "gtr_gla_path_for": ([I, I, I, I, I, I, I, I], I),
            "gtr_last_device_status": ([P, P], I),
            "gtr_gla_segment_chunks": ([I, I, I, I, I, I, I, I], I),
            "gtr_gla_segment_count": ([I, I, I, I, I, I, I, I], I),
            "gtr_gla_fwd_noalloc": ([P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P], I),
            "gtr_gate_packed_bytes": ([], Z),
            "gtr_gate_pack": ([P, P, I, I, I, I, I, P, Z, P], I),
            "gtr_gate_fwd_packed": ([P, I, P, P, P, I, I, I, I, I, I, F, P], I),
            "gtr_gla_fwd_gated": ([P, I, P, P, I, I, F, P, P, P, P, P, P, P,
                                   I, I, I, I, I, I, I, I, I, P], I),
            "gtr_gla_fwd_gated_timed": ([P, I, P, P, I, I, F, P, P, P, P, P, P, P,
                                         I, I, I, I, I, I, I, I, I, P, P], I),
            "gtr_mixer_in_proj": ([P, P, P, P, P, P, I, I, I, I, I, I, I, P], I),
            "gtr_mixer_out_proj": ([P, P, P, ctypes.c_longlong, I, I, I, P], I),
            "gtr_sswiglu_mix": ([P, P, P, P, I, I, I, I, I, I, P], I),
            "gtr_sswiglu_fwd": ([P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P], I),
            "gtr_stack_workspace_bytes": ([I, I, I, I, I, I, I, I], Z),
            "gtr_stack_fwd": ([P, P, I, P, I, I, I, I, I, I, I, I, F, I, I, P, Z, P], I),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
        return lib


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        msg = load().gtr_status_string(rc).decode()
        raise GtrError(fn, rc, msg)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, shape=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def gate_fwd(x: torch.Tensor, w_down: torch.Tensor, w_up: torch.Tensor,
             bias: Optional[torch.Tensor], H: int, dk: int, tau: float = 16.0,
             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """g = logsigmoid(x W_down W_up + bias) / tau as [B, T, H, dk] fp32 (``gtr_gate_fwd``)."""
    _need(x, "x")
    if x.dim() != 3:
        raise ValueError("x must be [B, T, d_model]")
    B, T, dm = x.shape
    rank = w_down.shape[1]
    _need(w_down, "w_down", torch.float32, (dm, rank))
    _need(w_up, "w_up", torch.float32, (rank, H * dk))
    if bias is not None:
        _need(bias, "bias", torch.float32, (H * dk,))
    if out is None:
        out = torch.empty(B, T, H, dk, device=x.device, dtype=torch.float32)
    _need(out, "out", torch.float32, (B, T, H, dk))
    rc = load().gtr_gate_fwd(_ptr(x), DTYPE_IDS[x.dtype], _ptr(w_down), _ptr(w_up), _ptr(bias),
                             _ptr(out), B, T, dm, rank, H, dk, float(tau), _stream(stream))
    _check("gtr_gate_fwd", rc)
    return out


def gate_pack(w_down: torch.Tensor, w_up: torch.Tensor, x_dtype: torch.dtype, H: int, dk: int,
              out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Packed gate weights for ``gate_fwd_packed`` (``gtr_gate_pack``): a uint8 device tensor."""
    dm, rank = w_down.shape
    _need(w_down, "w_down", torch.float32, (dm, rank))
    _need(w_up, "w_up", torch.float32, (rank, H * dk))
    nbytes = int(load().gtr_gate_packed_bytes())
    if out is None:
        out = torch.empty(nbytes, device=w_down.device, dtype=torch.uint8)
    rc = load().gtr_gate_pack(_ptr(w_down), _ptr(w_up), DTYPE_IDS[x_dtype], dm, rank, H, dk,
                              _ptr(out), out.numel(), _stream(stream))
    _check("gtr_gate_pack", rc)
    return out


def gate_fwd_packed(x: torch.Tensor, packed: torch.Tensor, bias: Optional[torch.Tensor], rank: int,
                    H: int, dk: int, tau: float = 16.0, out: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """``gate_fwd`` with weights packed by ``gate_pack`` (``gtr_gate_fwd_packed``)."""
    _need(x, "x")
    if x.dim() != 3:
        raise ValueError("x must be [B, T, d_model]")
    B, T, dm = x.shape
    if packed.dtype != torch.uint8 or packed.device != x.device:
        raise ValueError("packed must be a uint8 tensor on x's device")
    if bias is not None:
        _need(bias, "bias", torch.float32, (H * dk,))
    if out is None:
        out = torch.empty(B, T, H, dk, device=x.device, dtype=torch.float32)
    _need(out, "out", torch.float32, (B, T, H, dk))
    rc = load().gtr_gate_fwd_packed(_ptr(x), DTYPE_IDS[x.dtype], _ptr(packed), _ptr(bias), _ptr(out),
                                    B, T, dm, rank, H, dk, float(tau), _stream(stream))
    _check("gtr_gate_fwd_packed", rc)
    return out


def _gla_check(q, k, v, g, z, w, out, grid_h, grid_w):
    for name, t in (("q", q), ("k", k), ("v", v), ("z", z)):
        _need(t, name, q.dtype)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if T != grid_h * grid_w:
        raise ValueError(f"T={T} != grid_h*grid_w={grid_h * grid_w}")
    _need(k, "k", q.dtype, (B, T, H, dk))
    _need(v, "v", q.dtype, (B, T, H, dv))
    _need(z, "z", q.dtype, (B, T, H, dv))
    _need(g, "g", torch.float32, (B, T, H, dk))
    if w is not None:
        _need(w, "w", torch.float32, (dv,))
    if out is None:
        out = torch.empty(B, T, H, dv, device=q.device, dtype=q.dtype)
    _need(out, "out", q.dtype, (B, T, H, dv))
    return B, T, H, dk, dv, out


def gla_fwd(q, k, v, g, z, w=None, *, grid_h: int, grid_w: int, direction: str = "LR",
            chunk: int = 64, out: Optional[torch.Tensor] = None, stream=None,
            events: Optional[Sequence] = None) -> torch.Tensor:
    """y = RMSNorm(o) * w * SiLU(z) of the Key-only GLA (``gtr_gla_fwd``).

    q, k: [B, T, H, dk]; v, z: [B, T, H, dv] (one dtype); g: [B, T, H, dk] fp32;
    w: [dv] fp32 or None.  ``events`` (4 torch.cuda.Event or None) are recorded
    around the three stages on the launch stream (``gtr_gla_fwd_timed``).
    """
    B, T, H, dk, dv, out = _gla_check(q, k, v, g, z, w, out, grid_h, grid_w)
    lib = load()
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(z), _ptr(w), _ptr(out), B, H, grid_h, grid_w,
            dk, dv, DIR_IDS[direction], int(chunk), DTYPE_IDS[q.dtype], _stream(stream))
    if events is None:
        _check("gtr_gla_fwd", lib.gtr_gla_fwd(*args))
    else:
        arr = (ctypes.c_void_p * 4)(*[None if e is None else e.cuda_event for e in events])
        _check("gtr_gla_fwd_timed", lib.gtr_gla_fwd_timed(*args, arr))
    return out


def gla_fwd_gated(x, packed, bias, q, k, v, z, w=None, *, tau: float, grid_h: int, grid_w: int,
                  direction: str = "LR", chunk: int = 64, rank: int = 16,
                  g_out: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                  stream=None, events: Optional[Sequence] = None):
    """Gate projection and GLA forward in one call (``gtr_gla_fwd_gated``).

    x: [B, T, d_model] 16-bit; packed: ``gate_pack(w_down, w_up, x.dtype, H, dk)``;
    bias: [H*dk] fp32 or None; q, k, v, z, w as in :func:`gla_fwd`.  Returns
    (out, g_out) with g_out = logsigmoid(x W_down W_up + bias)/tau [B, T, H, dk]
    fp32.  ``events`` (5 torch.cuda.Event or None) are recorded before the gate
    and after each of its four kernels (``gtr_gla_fwd_gated_timed``).
    """
    _need(x, "x")
    if x.dim() != 3:
        raise ValueError("x must be [B, T, d_model]")
    if packed.dtype != torch.uint8 or packed.device != x.device:
        raise ValueError("packed must be a uint8 tensor on x's device")
    B, T, H, dk = q.shape
    if g_out is None:
        g_out = torch.empty(B, T, H, dk, device=q.device, dtype=torch.float32)
    B, T, H, dk, dv, out = _gla_check(q, k, v, g_out, z, w, out, grid_h, grid_w)
    if tuple(x.shape[:2]) != (B, T):
        raise ValueError(f"x must be [B={B}, T={T}, d_model], got {tuple(x.shape)}")
    if bias is not None:
        _need(bias, "bias", torch.float32, (H * dk,))
    lib = load()
    args = (_ptr(x), DTYPE_IDS[x.dtype], _ptr(packed), _ptr(bias), x.shape[2], int(rank), float(tau),
            _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(w), _ptr(g_out), _ptr(out), B, H, grid_h, grid_w,
            dk, dv, DIR_IDS[direction], int(chunk), DTYPE_IDS[q.dtype], _stream(stream))
    if events is None:
        _check("gtr_gla_fwd_gated", lib.gtr_gla_fwd_gated(*args))
    else:
        arr = (ctypes.c_void_p * 5)(*[None if e is None else e.cuda_event for e in events])
        _check("gtr_gla_fwd_gated_timed", lib.gtr_gla_fwd_gated_timed(*args, arr))
    return out, g_out


def mixer_in_proj(x, w_in, H: int, dk: int, dv: Optional[int] = None, stream=None):
    """q, k, v, z = x W_q, x W_k, x W_v, x W_z (``gtr_mixer_in_proj``).

    x: [B, T, d_model] 16-bit; w_in: [d_model, 2 H dk + 2 H dv] of x's dtype,
    column blocks W_q | W_k | W_v | W_z.  Returns q, k [B, T, H, dk] and v, z
    [B, T, H, dv] in x's dtype."""
    dv = dk if dv is None else dv
    _need(x, "x")
    if x.dim() != 3:
        raise ValueError("x must be [B, T, d_model]")
    B, T, dm = x.shape
    _need(w_in, "w_in", x.dtype, (dm, 2 * H * dk + 2 * H * dv))
    if dv == dk:   # one buffer: the four outputs equally spaced (one batched product)
        q, k, v, z = torch.empty(4, B, T, H, dk, device=x.device, dtype=x.dtype).unbind(0)
    else:
        q = torch.empty(B, T, H, dk, device=x.device, dtype=x.dtype)
        k = torch.empty_like(q)
        v = torch.empty(B, T, H, dv, device=x.device, dtype=x.dtype)
        z = torch.empty_like(v)
    rc = load().gtr_mixer_in_proj(_ptr(x), _ptr(w_in), _ptr(q), _ptr(k), _ptr(v), _ptr(z), B, T, dm, H, dk,
                                  dv, DTYPE_IDS[x.dtype], _stream(stream))
    _check("gtr_mixer_in_proj", rc)
    return q, k, v, z


def mixer_out_proj(y, w_out, stream=None):
    """out = y w_out (``gtr_mixer_out_proj``): y [..., d_in], w_out [d_in, d_out], one 16-bit dtype."""
    _need(y, "y")
    d_in = y.shape[-1]
    _need(w_out, "w_out", y.dtype)
    if w_out.dim() != 2 or w_out.shape[0] != d_in:
        raise ValueError(f"w_out must be [{d_in}, d_out]")
    d_out = w_out.shape[1]
    out = torch.empty(*y.shape[:-1], d_out, device=y.device, dtype=y.dtype)
    N = y.numel() // d_in if d_in else 0
    rc = load().gtr_mixer_out_proj(_ptr(y), _ptr(w_out), _ptr(out), N, d_in, d_out, DTYPE_IDS[y.dtype],
                                   _stream(stream))
    _check("gtr_mixer_out_proj", rc)
    return out


def _conv_check(conv_w, conv_b, C: int, ksize: int = 3):
    _need(conv_w, "conv_w", torch.float32, (ksize, ksize, C))
    if conv_b is not None:
        _need(conv_b, "conv_b", torch.float32, (C,))


def sswiglu_mix(u, conv_w, conv_b=None, *, grid_h: int, grid_w: int, out=None, stream=None):
    """The Spatial SwiGLU hidden activation (``gtr_sswiglu_mix``): u [B, T, 2C]
    16-bit (gate channels first, value channels last, T = grid_h * grid_w in
    grid order), conv_w [3, 3, C] fp32, conv_b [C] fp32 or None ->
    h = SiLU(u_gate) * (depthwise 3x3 convolution of u_value on the grid + conv_b)
    as [B, T, C] in u's dtype."""
    _need(u, "u")
    if u.dim() != 3 or u.shape[1] != grid_h * grid_w or u.shape[2] % 2:
        raise ValueError("u must be [B, grid_h * grid_w, 2C]")
    B, T, C2 = u.shape
    C = C2 // 2
    _conv_check(conv_w, conv_b, C, conv_w.shape[0] if conv_w.dim() == 3 else 3)
    if out is None:
        out = torch.empty(B, T, C, device=u.device, dtype=u.dtype)
    _need(out, "out", u.dtype, (B, T, C))
    rc = load().gtr_sswiglu_mix(_ptr(u), _ptr(conv_w), _ptr(conv_b), _ptr(out), B, grid_h, grid_w, C,
                                conv_w.shape[0], DTYPE_IDS[u.dtype], _stream(stream))
    _check("gtr_sswiglu_mix", rc)
    return out


def sswiglu_fwd(x, w_in, conv_w, conv_b, w_out, *, grid_h: int, grid_w: int, scratch=None, stream=None):
    """The Spatial SwiGLU block (``gtr_sswiglu_fwd``): x [B, T, d_model] 16-bit,
    w_in [d_model, 2C] and w_out [C, d_model] of x's dtype, conv_w [3, 3, C] and
    conv_b [C] fp32 -> y [B, T, d_model].  ``scratch`` is an optional (u, h)
    pair of [B, T, 2C] and [B, T, C] tensors that receive the expansion and the
    hidden activation; they are allocated when not given."""
    _need(x, "x")
    if x.dim() != 3 or x.shape[1] != grid_h * grid_w:
        raise ValueError("x must be [B, grid_h * grid_w, d_model]")
    B, T, dm = x.shape
    _need(w_in, "w_in", x.dtype)
    if w_in.dim() != 2 or w_in.shape[0] != dm or w_in.shape[1] % 2:
        raise ValueError(f"w_in must be [{dm}, 2C]")
    C = w_in.shape[1] // 2
    _need(w_out, "w_out", x.dtype, (C, dm))
    _conv_check(conv_w, conv_b, C, conv_w.shape[0] if conv_w.dim() == 3 else 3)
    if scratch is None:
        scratch = (torch.empty(B, T, 2 * C, device=x.device, dtype=x.dtype),
                   torch.empty(B, T, C, device=x.device, dtype=x.dtype))
    u, h = scratch
    _need(u, "u", x.dtype, (B, T, 2 * C))
    _need(h, "h", x.dtype, (B, T, C))
    y = torch.empty(B, T, dm, device=x.device, dtype=x.dtype)
    rc = load().gtr_sswiglu_fwd(_ptr(x), _ptr(w_in), _ptr(conv_w), _ptr(conv_b), _ptr(w_out), _ptr(u), _ptr(h),
                                _ptr(y), B, grid_h, grid_w, dm, C, conv_w.shape[0], DTYPE_IDS[x.dtype],
                                _stream(stream))
    _check("gtr_sswiglu_fwd", rc)
    return y


def stack_workspace_bytes(B: int, grid_h: int, grid_w: int, d_model: int, H: int, dk: int, dv: int,
                          hidden: int) -> int:
    return int(load().gtr_stack_workspace_bytes(B, grid_h, grid_w, d_model, H, dk, dv, hidden))


def stack_weights(blocks, dtype: torch.dtype, H: int, dk: int, device, stream=None):
    """Device copies of host block weights (dicts with the keys of
    ``BLOCK_FIELDS`` except gate_packed, plus w_down and w_up), with each
    block's gate weights packed by ``gtr_gate_pack`` for x of ``dtype``."""
    out = []
    for p in blocks:
        d = {n: (None if p.get(n) is None else p[n].to(device).contiguous())
             for n in BLOCK_FIELDS if n != "gate_packed"}
        d["gate_packed"] = gate_pack(p["w_down"].to(device).contiguous(), p["w_up"].to(device).contiguous(),
                                     dtype, H, dk, stream=stream)
        out.append(d)
    return out


def stack_fwd(x, blocks, *, grid_h: int, grid_w: int, H: int, dk: int, dv: int, dtype: torch.dtype,
              tau: float = 16.0, chunk: int = 64, directions: Optional[Sequence[str]] = None,
              workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """``gtr_stack_fwd``: the blocks applied in order to the fp32 residual
    stream x [B, grid_h*grid_w, d_model] in place (returns x).  ``blocks`` are
    dicts of device tensors (``stack_weights``); every other activation is in
    ``dtype``; ``workspace`` is a uint8 device tensor of at least
    ``stack_workspace_bytes`` bytes, allocated when not given."""
    _need(x, "x", torch.float32)
    if x.dim() != 3 or x.shape[1] != grid_h * grid_w:
        raise ValueError("x must be [B, grid_h * grid_w, d_model]")
    B, T, dm = x.shape
    if not blocks:
        return x
    hidden = blocks[0]["w_p"].shape[0]
    arr = (BlockWeights * len(blocks))()
    for i, p in enumerate(blocks):
        for n in BLOCK_FIELDS:
            t = p.get(n)
            if t is not None:
                _need(t, n)
                setattr(arr[i], n, t.data_ptr())
    dirs = None
    if directions is not None:
        if len(directions) != len(blocks):
            raise ValueError("one direction per block")
        dirs = (ctypes.c_int * len(blocks))(*[DIR_IDS[d] for d in directions])
    need = stack_workspace_bytes(B, grid_h, grid_w, dm, H, dk, dv, hidden)
    if workspace is None:
        workspace = torch.empty(need, device=x.device, dtype=torch.uint8)
    rc = load().gtr_stack_fwd(_ptr(x), arr, len(blocks), dirs, B, grid_h, grid_w, dm, H, dk, dv, hidden,
                              float(tau), int(chunk), DTYPE_IDS[dtype], _ptr(workspace), workspace.numel(),
                              _stream(stream))
    _check("gtr_stack_fwd", rc)
    return x


def gla_fwd_noalloc(q, k, v, g, z, w=None, *, grid_h: int, grid_w: int, direction: str = "LR",
                    chunk: int = 64, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """``gtr_gla_fwd_noalloc``: the result of :func:`gla_fwd` without any device allocation
    by the library (its scratch is a fixed static device array; see include/gtr_gla.h).
    Raises GtrError with status -4 when the problem needs more than that scratch."""
    B, T, H, dk, dv, out = _gla_check(q, k, v, g, z, w, out, grid_h, grid_w)
    rc = load().gtr_gla_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(z), _ptr(w), _ptr(out),
                                    B, H, grid_h, grid_w, dk, dv, DIR_IDS[direction], int(chunk),
                                    DTYPE_IDS[q.dtype], _stream(stream))
    _check("gtr_gla_fwd_noalloc", rc)
    return out


def chunk_states(k, v, g, *, grid_h: int, grid_w: int, direction: str = "LR", chunk: int = 64,
                 stream=None) -> torch.Tensor:
    """State each chunk ends with: [B, H, ceil(T/chunk), dk, dv] fp32 (``gtr_gla_chunk_states``)."""
    _need(k, "k")
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    _need(v, "v", k.dtype, (B, T, H, dv))
    _need(g, "g", torch.float32, (B, T, H, dk))
    nc = (T + chunk - 1) // chunk
    st = torch.empty(B, H, nc, dk, dv, device=k.device, dtype=torch.float32)
    rc = load().gtr_gla_chunk_states(_ptr(k), _ptr(v), _ptr(g), _ptr(st), B, H, grid_h, grid_w,
                                     dk, dv, DIR_IDS[direction], int(chunk), DTYPE_IDS[k.dtype],
                                     _stream(stream))
    _check("gtr_gla_chunk_states", rc)
    return st


def set_path(path: str) -> None:
    _check("gtr_gla_set_path", load().gtr_gla_set_path(PATH_IDS[path]))


def path_for(B, H, grid_h, grid_w, dk, dv, chunk, dtype) -> str:
    rc = load().gtr_gla_path_for(B, H, grid_h, grid_w, dk, dv, chunk, DTYPE_IDS[dtype])
    if rc < 0:
        _check("gtr_gla_path_for", rc)
    return PATH_NAMES[rc]


def workspace_bytes(B, H, grid_h, grid_w, dk, dv, chunk, dtype) -> int:
    return int(load().gtr_gla_workspace_bytes(B, H, grid_h, grid_w, dk, dv, chunk, DTYPE_IDS[dtype]))


def segment_chunks(B, H, grid_h, grid_w, dk, dv, chunk, dtype) -> int:
    rc = load().gtr_gla_segment_chunks(B, H, grid_h, grid_w, dk, dv, chunk, DTYPE_IDS[dtype])
    if rc < 0:
        _check("gtr_gla_segment_chunks", rc)
    return rc


def segment_count(B, H, grid_h, grid_w, dk, dv, chunk, dtype) -> int:
    rc = load().gtr_gla_segment_count(B, H, grid_h, grid_w, dk, dv, chunk, DTYPE_IDS[dtype])
    if rc < 0:
        _check("gtr_gla_segment_count", rc)
    return rc


def set_workspace(buf: Optional[torch.Tensor]) -> None:
    if buf is None:
        _check("gtr_gla_set_workspace", load().gtr_gla_set_workspace(None, 0))
    else:
        _need(buf, "workspace")
        nbytes = buf.numel() * buf.element_size()
        _check("gtr_gla_set_workspace", load().gtr_gla_set_workspace(_ptr(buf), nbytes))


def device_status(stream=None):
    """(status, exact_chunks): synchronises the stream and clears the device record."""
    counters = (ctypes.c_ulonglong * 2)()
    rc = load().gtr_last_device_status(_stream(stream), counters)
    return rc, int(counters[0]), int(counters[1])

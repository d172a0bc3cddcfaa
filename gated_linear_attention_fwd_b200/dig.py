"""Thin ctypes binding of libdig.so (include/dig.h).

Argument marshalling only: tensors are passed as raw device pointers with their
sizes and the current CUDA stream; every step of the computation runs in the
library's sm_100a kernels.  Importing this module fails loudly when libdig.so
has not been built -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdig.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "dig.h")

if not os.path.exists(LIB_PATH):
    raise ImportError("libdig.so is not built; run `python -m gated_linear_attention_fwd_b200.build` "
                      "(or __graft_entry__.build()) first")

lib = ctypes.CDLL(LIB_PATH)

DIG_OK = 0
DIG_ERR_INVALID_ARGUMENT = 1
DIG_ERR_UNSUPPORTED = 2
DIG_ERR_MISALIGNED = 3
DIG_ERR_WORKSPACE_TOO_SMALL = 4
DIG_ERR_CUDA = 5
DIG_ERR_DEVICE_TIMEOUT = 6
DIG_ERR_GATE_RANGE = 7

DIG_F32 = 0
DIG_BF16 = 1

SCAN_ROW_FWD, SCAN_ROW_REV, SCAN_COL_FWD, SCAN_COL_REV = 0, 1, 2, 3

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t

lib.dig_gla_supported.restype = _i
lib.dig_gla_supported.argtypes = [_i, _i]
lib.dig_gla_workspace_bytes.restype = _sz
lib.dig_gla_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i]
lib.dig_gla_fwd.restype = _i
lib.dig_gla_fwd.argtypes = [_vp, _vp, _vp, _vp, _i, _f, _vp, _vp, _vp, _f, _vp,
                            _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]
lib.dig_gla_fwd_noalloc.restype = _i
lib.dig_gla_fwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i, _f, _vp, _vp, _vp, _f, _vp,
                                    _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp]
lib.dig_gla_bwd.restype = _i
lib.dig_gla_bwd.argtypes = [_vp, _vp, _vp, _vp, _i, _f, _vp, _vp, _vp, _vp, _vp,
                            _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]
lib.dig_gla_bwd_saved.restype = _i
lib.dig_gla_bwd_saved.argtypes = [_vp, _vp, _vp, _vp, _i, _f, _vp, _vp, _vp, _vp, _vp,
                                  _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp, _sz, _vp]
lib.dig_gla_ext_workspace_bytes.restype = _sz
lib.dig_gla_ext_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i]
lib.dig_gla_fwd_ext.restype = _i
lib.dig_gla_fwd_ext.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _f, _vp, _vp, _vp, _vp, _f, _vp, _vp,
                                _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]
lib.dig_gla_bwd_ext.restype = _i
lib.dig_gla_bwd_ext.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _f, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]
lib.dig_srem_reorient_dwconv.restype = _i
lib.dig_srem_reorient_dwconv.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]
lib.dig_srem_reorient_dwconv_bwd.restype = _i
lib.dig_srem_reorient_dwconv_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]
lib.dig_epilogue_bwd.restype = _i
lib.dig_epilogue_bwd.argtypes = [_vp, _vp, _vp, _f, _vp, _vp, _vp, _vp, ctypes.c_longlong, _i, _i, _i, _vp]
lib.dig_gate_proj_fwd.restype = _i
lib.dig_gate_proj_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_longlong, _i, _i, _i, _i, _vp]
lib.dig_gate_proj_bwd.restype = _i
lib.dig_gate_proj_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp, ctypes.c_longlong,
                                  _i, _i, _i, _i, _i, _vp]
lib.dig_block_rmsnorm_modulate.restype = _i
lib.dig_block_rmsnorm_modulate.argtypes = [_vp, _vp, _vp, ctypes.c_longlong, _f, _vp, _i, ctypes.c_longlong, _i, _vp]
lib.dig_block_gated_add.restype = _i
lib.dig_block_gated_add.argtypes = [_vp, _vp, ctypes.c_longlong, _vp, _i, ctypes.c_longlong, _i, _vp]
lib.dig_block_activation.restype = _i
lib.dig_block_activation.argtypes = [_vp, ctypes.c_longlong, _i, _vp]
lib.dig_read_status.restype = _i
lib.dig_read_status.argtypes = [_vp, _vp]
lib.dig_status_string.restype = ctypes.c_char_p
lib.dig_status_string.argtypes = [_i]
lib.dig_last_error.restype = ctypes.c_char_p
lib.dig_last_error.argtypes = []


class DigError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.dig_last_error().decode(errors="replace")
        super().__init__("%s: %s (%d)%s" % (where, lib.dig_status_string(status).decode(), status,
                                            (": " + msg) if msg else ""))


def header_functions() -> list[str]:
    """Names of the functions include/dig.h declares."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dig_[a-z0-9_]+)\s*\(", src)))


def _code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return DIG_F32
    if dt == torch.bfloat16:
        return DIG_BF16
    raise TypeError("unsupported dtype %s (float32 or bfloat16)" % dt)


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(st, where):
    if st != DIG_OK:
        raise DigError(st, where)


def gla_workspace_bytes(B, H, L, d_k, d_v, backward=False, gate_heads=1) -> int:
    return int(lib.dig_gla_workspace_bytes(B, H, gate_heads, L, d_k, d_v, 1 if backward else 0))


def new_workspace(B, H, L, d_k, d_v, backward=False, device="cuda", gate_heads=1) -> torch.Tensor:
    """A zero-filled workspace (uint8) sized for dig_gla_fwd / dig_gla_bwd."""
    n = gla_workspace_bytes(B, H, L, d_k, d_v, backward, gate_heads)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def dig_gla_fwd(q, k, v, z, inv_tau, o, grid_h, grid_w, scan_mode, workspace,
                r=None, gamma=None, eps=1e-5, y=None, stream=None):
    """q,k [B,L,H,dk]; v,o [B,L,H,dv]; z [B,L,gate_heads,dk] fp32 (see include/dig.h)."""
    B, L, H, dk = q.shape
    dv = v.shape[3]
    st = lib.dig_gla_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(z), z.shape[2], float(inv_tau), _ptr(o),
                         _ptr(r), _ptr(gamma), float(eps), _ptr(y),
                         B, H, L, dk, dv, grid_h, grid_w, scan_mode, _code(q.dtype), _code(o.dtype),
                         _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "dig_gla_fwd")


def dig_gla_fwd_noalloc(q, k, v, z, inv_tau, o, grid_h, grid_w, scan_mode, r=None, gamma=None, eps=1e-5, y=None,
                        device_status=None, stream=None):
    """dig_gla_fwd on the library's built-in scratch (no workspace argument; for
    callers that cannot allocate device memory).  device_status: optional int32
    CUDA tensor receiving the call's device status word."""
    B, L, H, dk = q.shape
    dv = v.shape[3]
    st = lib.dig_gla_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(z), z.shape[2], float(inv_tau), _ptr(o),
                                 _ptr(r), _ptr(gamma), float(eps), _ptr(y),
                                 B, H, L, dk, dv, grid_h, grid_w, scan_mode, _code(q.dtype), _code(o.dtype),
                                 _ptr(device_status), _stream(stream))
    _check(st, "dig_gla_fwd_noalloc")


def dig_gla_bwd(q, k, v, z, inv_tau, dO, dq, dk, dv, dlog_alpha, grid_h, grid_w, scan_mode, workspace,
                stream=None):
    B, L, H, d_k = q.shape
    d_v = v.shape[3]
    st = lib.dig_gla_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(z), z.shape[2], float(inv_tau), _ptr(dO),
                         _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlog_alpha),
                         B, H, L, d_k, d_v, grid_h, grid_w, scan_mode, _code(q.dtype), _code(dq.dtype),
                         _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "dig_gla_bwd")


def dig_gla_bwd_saved(q, k, v, z, inv_tau, dO, dq, dk, dv, dlog_alpha, grid_h, grid_w, scan_mode, fwd_workspace,
                      workspace, stream=None):
    """dig_gla_bwd reusing the records dig_gla_fwd left in fwd_workspace (same inputs, see include/dig.h)."""
    B, L, H, d_k = q.shape
    d_v = v.shape[3]
    st = lib.dig_gla_bwd_saved(_ptr(q), _ptr(k), _ptr(v), _ptr(z), z.shape[2], float(inv_tau), _ptr(dO),
                               _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlog_alpha),
                               B, H, L, d_k, d_v, grid_h, grid_w, scan_mode, _code(q.dtype), _code(dq.dtype),
                               _ptr(fwd_workspace), fwd_workspace.numel() * fwd_workspace.element_size(),
                               _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "dig_gla_bwd_saved")


def new_ext_workspace(B, H, L, d_k, d_v, dtype=torch.bfloat16, backward=False, device="cuda",
                      gate_heads=1) -> torch.Tensor:
    """A zero-filled workspace (uint8) sized for dig_gla_fwd_ext / dig_gla_bwd_ext."""
    n = int(lib.dig_gla_ext_workspace_bytes(B, H, gate_heads, L, d_k, d_v, _code(dtype), 1 if backward else 0))
    if n == 0:
        raise ValueError("unsupported shape for the extended GLA entry points")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def dig_gla_fwd_ext(q, k, v, z, inv_tau, o, grid_h, grid_w, scan_mode, workspace, zb=None, S0=None,
                    S_final=None, r=None, gamma=None, eps=1e-5, y=None, stream=None):
    """GLA with a value gate (zb [B,L,gate_heads,dv] fp32 logits) and state input /
    output (S0, S_final [B,H,dk,dv] fp32); see include/dig.h."""
    B, L, H, dk = q.shape
    dv = v.shape[3]
    st = lib.dig_gla_fwd_ext(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(zb), z.shape[2], float(inv_tau), _ptr(S0),
                             _ptr(o), _ptr(r), _ptr(gamma), float(eps), _ptr(y), _ptr(S_final),
                             B, H, L, dk, dv, grid_h, grid_w, scan_mode, _code(q.dtype), _code(o.dtype),
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "dig_gla_fwd_ext")


def dig_gla_bwd_ext(q, k, v, z, inv_tau, dO, dq, dk, dv, dlog_alpha, grid_h, grid_w, scan_mode, workspace,
                    zb=None, S0=None, o=None, dS_final=None, dlog_beta=None, dS0=None, stream=None):
    """Gradients for dig_gla_fwd_ext (see include/dig.h); o is the forward's output,
    needed for dlog_beta."""
    B, L, H, d_k = q.shape
    d_v = v.shape[3]
    st = lib.dig_gla_bwd_ext(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(zb), z.shape[2], float(inv_tau), _ptr(S0),
                             _ptr(o), _ptr(dO), _ptr(dS_final), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlog_alpha),
                             _ptr(dlog_beta), _ptr(dS0),
                             B, H, L, d_k, d_v, grid_h, grid_w, scan_mode, _code(q.dtype), _code(dq.dtype),
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "dig_gla_bwd_ext")


def dig_srem_reorient_dwconv(x, w, bias, y, scan_mode, stream=None):
    """x [B,Hg,Wg,C] grid order; w [C,3,3] fp32; bias [C] fp32 or None; y [B,L,C] scan order."""
    B, Hg, Wg, C = x.shape
    st = lib.dig_srem_reorient_dwconv(_ptr(x), _ptr(w), _ptr(bias), _ptr(y), B, Hg, Wg, C, scan_mode,
                                      _code(x.dtype), _code(y.dtype), _stream(stream))
    _check(st, "dig_srem_reorient_dwconv")


def dig_srem_reorient_dwconv_bwd(x, w, dY, dx, scan_mode, dw=None, dbias=None, stream=None):
    """x, dx [B,Hg,Wg,C] grid order; w [C,3,3] fp32; dY [B,L,C] scan order; dw [C,3,3], dbias [C] fp32 or None."""
    B, Hg, Wg, C = dx.shape
    st = lib.dig_srem_reorient_dwconv_bwd(_ptr(x), _ptr(w), _ptr(dY), _ptr(dx), _ptr(dw), _ptr(dbias),
                                          B, Hg, Wg, C, scan_mode, _code(dY.dtype), _code(dx.dtype), _stream(stream))
    _check(st, "dig_srem_reorient_dwconv_bwd")


def dig_epilogue_bwd(o, r, dY, d_o, d_r, gamma=None, eps=1e-5, d_gamma=None, stream=None):
    """o, r, dY [..., d_v] (same dtype); d_o, d_r [..., d_v]; gamma, d_gamma [d_v] fp32 or None."""
    d_v = o.shape[-1]
    rows = o.numel() // d_v if d_v else 0
    st = lib.dig_epilogue_bwd(_ptr(o), _ptr(r), _ptr(gamma), float(eps), _ptr(dY), _ptr(d_o), _ptr(d_r),
                              _ptr(d_gamma), rows, d_v, _code(o.dtype), _code(d_o.dtype), _stream(stream))
    _check(st, "dig_epilogue_bwd")


def dig_gate_proj_fwd(x, W1, W2, z, b=None, u=None, stream=None):
    """x [..., D]; W1 [D,R], W2 [R,d_k] fp32; z [..., d_k] fp32; b [d_k] or None; u [..., R] fp32 or None."""
    D, R = W1.shape
    d_k = W2.shape[1]
    rows = x.numel() // D
    st = lib.dig_gate_proj_fwd(_ptr(x), _ptr(W1), _ptr(W2), _ptr(b), _ptr(z), _ptr(u), rows, D, R, d_k,
                               _code(x.dtype), _stream(stream))
    _check(st, "dig_gate_proj_fwd")


def dig_gate_proj_bwd(x, W1, W2, u, z, dlog_alpha, inv_tau, dx, dW1, dW2, db=None, stream=None):
    """Gradients of the gate projection from d log(alpha) (see include/dig.h)."""
    D, R = W1.shape
    d_k = W2.shape[1]
    rows = x.numel() // D
    st = lib.dig_gate_proj_bwd(_ptr(x), _ptr(W1), _ptr(W2), _ptr(u), _ptr(z), _ptr(dlog_alpha), float(inv_tau),
                               _ptr(dx), _ptr(dW1), _ptr(dW2), _ptr(db), rows, D, R, d_k, _code(x.dtype),
                               _code(dx.dtype), _stream(stream))
    _check(st, "dig_gate_proj_bwd")


def _mod_stride(t):
    """Row stride (in values) of a [B, D] modulation slice."""
    return t.stride(0)


def dig_block_rmsnorm_modulate(x, shift, scale, y, eps=1e-6, stream=None):
    """y = RMSNorm(x) * (1 + scale[b]) + shift[b]; x, y [B, rows, D] bf16; shift, scale
    [B, D] fp32 (rows of one [B, 6 D] tensor may be passed as slices)."""
    B, rows, D = x.shape
    if shift.stride(1) != 1 or scale.stride(1) != 1 or shift.stride(0) != scale.stride(0):
        raise ValueError("shift and scale must be row slices of one tensor")
    st = lib.dig_block_rmsnorm_modulate(_ptr(x), ctypes.c_void_p(shift.data_ptr()), ctypes.c_void_p(scale.data_ptr()),
                                        _mod_stride(shift), float(eps), _ptr(y), B, rows, D, _stream(stream))
    _check(st, "dig_block_rmsnorm_modulate")


def dig_block_gated_add(x, gate, y, stream=None):
    """x += gate[b] * y; x, y [B, rows, D] bf16; gate [B, D] fp32 (a row slice)."""
    B, rows, D = x.shape
    if gate.stride(1) != 1:
        raise ValueError("gate must have unit stride along D")
    st = lib.dig_block_gated_add(_ptr(x), ctypes.c_void_p(gate.data_ptr()), _mod_stride(gate), _ptr(y), B, rows, D,
                                 _stream(stream))
    _check(st, "dig_block_gated_add")


def dig_block_activation(x, kind, stream=None):
    """In place on bf16 x: kind 0 SiLU, kind 1 GELU (tanh form)."""
    st = lib.dig_block_activation(_ptr(x), x.numel(), int(kind), _stream(stream))
    _check(st, "dig_block_activation")


def dig_read_status(workspace, stream=None) -> int:
    return int(lib.dig_read_status(_ptr(workspace), _stream(stream)))

"""fp64 CPU oracle of the DiG token mixer (GLA recurrence, backward, SREM, epilogue).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with the CUDA path and never imports it.

Every function takes numpy arrays (any float dtype; they are widened to fp64)
in the layouts documented in ``oracle.c`` and returns fp64 arrays.

Parity status of each function (what pins it is in tests/test_oracle_pins.py):
  gla_fwd        pinned: brute-force quadratic form, alpha==1 causal linear
                 attention, alpha->0 diagonal case, constant-gate closed form,
                 causality and linearity
  gla_fwd_ext    pinned: segment split (the second half started from the first half's
                 final state equals the whole run), the S0-only closed form
                 (k = 0), brute-force quadratic form with a value gate
  gla_bwd_ext    pinned: central finite differences of sum(o * dO) + sum(S_final * dSf)
                 in q, k, v, z, zb and S0, across checkpoint blocks
  gla_bwd        pinned: central finite differences of a scalar loss, and the
                 reverse-cumsum identity for d log(alpha)
  srem_dwconv    pinned: scipy.signal.correlate2d, identity kernel = pure
                 permutation, all-ones kernel on a constant grid (9/6/4)
  epilogue       pinned: unit RMS of the normalised row, Swish(0) = 0,
                 positive scale invariance
  epilogue_bwd   pinned: central finite differences of sum(dy * epilogue) in o, r
                 and gamma; d_o orthogonal to o when eps = 0 (scale invariance)
  gate_proj_fwd  pinned: numpy matmul (x @ W1) @ W2 + b; rank-one closed form
  gate_proj_bwd  pinned: central finite differences of sum(dla * inv_tau * logsigmoid(z))
                 in x, W1, W2 and b
  srem_dwconv_bwd pinned: adjoint identity <conv(x), dy> = <x, dx>; dw and dbias
                 from the forward conv with one-tap kernels / zero kernel
  scan_index     pinned: bijection, inverse restores the grid, transpose on
                 square grids, a hand-derived 3x4 fixture
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        L = ctypes.c_long
        lib.oracle_scan_index.restype = L
        lib.oracle_scan_index.argtypes = [ctypes.c_int, L, L, L]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_gla_fwd.restype = ctypes.c_int
        lib.oracle_gla_fwd.argtypes = [dp, dp, dp, dp, ctypes.c_int, ctypes.c_double, dp,
                                       L, L, L, L, L, L, L, ctypes.c_int]
        lib.oracle_gla_fwd_ext.restype = ctypes.c_int
        lib.oracle_gla_fwd_ext.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_double, dp, dp, dp,
                                           L, L, L, L, L, L, L, ctypes.c_int]
        lib.oracle_gla_bwd_ext.restype = ctypes.c_int
        lib.oracle_gla_bwd_ext.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_double, dp, dp, dp,
                                           dp, dp, dp, dp, dp, dp, L, L, L, L, L, L, L, ctypes.c_int]
        lib.oracle_gla_bwd.restype = ctypes.c_int
        lib.oracle_gla_bwd.argtypes = [dp, dp, dp, dp, ctypes.c_int, ctypes.c_double, dp,
                                       dp, dp, dp, dp, L, L, L, L, L, L, L, ctypes.c_int]
        lib.oracle_epilogue.restype = ctypes.c_int
        lib.oracle_epilogue.argtypes = [dp, dp, dp, ctypes.c_double, dp, L, L]
        lib.oracle_epilogue_bwd.restype = ctypes.c_int
        lib.oracle_epilogue_bwd.argtypes = [dp, dp, dp, ctypes.c_double, dp, dp, dp, dp, L, L]
        lib.oracle_srem_dwconv_bwd.restype = ctypes.c_int
        lib.oracle_srem_dwconv_bwd.argtypes = [dp, dp, dp, dp, dp, dp, L, L, L, L, ctypes.c_int]
        lib.oracle_gate_proj_fwd.restype = ctypes.c_int
        lib.oracle_gate_proj_fwd.argtypes = [dp, dp, dp, dp, dp, dp, L, L, L, L]
        lib.oracle_gate_proj_bwd.restype = ctypes.c_int
        lib.oracle_gate_proj_bwd.argtypes = [dp, dp, dp, dp, dp, ctypes.c_double, dp, dp, dp, dp, L, L, L, L]
        lib.oracle_srem_dwconv.restype = ctypes.c_int
        lib.oracle_srem_dwconv.argtypes = [dp, dp, dp, dp, L, L, L, L, ctypes.c_int]
        _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def scan_index(mode: int, grid_h: int, grid_w: int) -> np.ndarray:
    """perm[t] = grid index (row * grid_w + col) visited at scan position t."""
    lib = _load()
    L = grid_h * grid_w
    out = np.array([lib.oracle_scan_index(mode, grid_h, grid_w, t) for t in range(L)],
                   dtype=np.int64)
    if L and out.min() < 0:
        raise ValueError("bad scan mode %r" % (mode,))
    return out


def gla_fwd(q, k, v, z, inv_tau, grid_h, grid_w, mode):
    """o [B,L,H,dv] of the GLA recurrence.  q,k [B,L,H,dk]; v [B,L,H,dv];
    z [B,L,Hz,dk] gate logits with Hz in {1, H}."""
    q, k, v, z = _f64(q), _f64(k), _f64(v), _f64(z)
    B, L, H, dk = q.shape
    dv = v.shape[3]
    gh = z.shape[2]
    o = np.zeros((B, L, H, dv), dtype=np.float64)
    rc = _load().oracle_gla_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(z), gh, float(inv_tau), _ptr(o),
                                B, H, L, dk, dv, grid_h, grid_w, int(mode))
    if rc:
        raise ValueError("oracle_gla_fwd rejected the arguments (rc=%d)" % rc)
    return o


def gla_fwd_ext(q, k, v, z, inv_tau, Hg, Wg, mode, zb=None, S0=None):
    """The recurrence with a value gate and state I/O: G_t = alpha_t^T beta_t, beta from
    value-gate logits zb [B,L,Hz,dv] (None: beta = 1), initial state S0 [B,H,dk,dv]
    (None: 0).  Returns (o [B,L,H,dv], S_final [B,H,dk,dv])."""
    q, k, v, z = _f64(q), _f64(k), _f64(v), _f64(z)
    B, L, H, dk = q.shape
    dv = v.shape[3]
    gh = z.shape[2]
    zz = None if zb is None else _f64(zb)
    s0 = None if S0 is None else _f64(S0)
    o = np.zeros((B, L, H, dv), dtype=np.float64)
    sf = np.zeros((B, H, dk, dv), dtype=np.float64)
    rc = _load().oracle_gla_fwd_ext(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(zz), gh, float(inv_tau), _ptr(s0),
                                    _ptr(o), _ptr(sf), B, H, L, dk, dv, Hg, Wg, int(mode))
    if rc:
        raise ValueError("oracle_gla_fwd_ext rejected the arguments")
    return o, sf


def gla_bwd_ext(q, k, v, z, inv_tau, dO, Hg, Wg, mode, zb=None, S0=None, dSf=None):
    """Gradients of sum(o * dO) + sum(S_final * dSf) for gla_fwd_ext.  Returns
    (dq, dk, dv, dlogalpha, dlogbeta or None, dS0 [B,H,dk,dv])."""
    q, k, v, z, dO = _f64(q), _f64(k), _f64(v), _f64(z), _f64(dO)
    B, L, H, dk = q.shape
    dv = v.shape[3]
    gh = z.shape[2]
    zz = None if zb is None else _f64(zb)
    s0 = None if S0 is None else _f64(S0)
    dsf = None if dSf is None else _f64(dSf)
    dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dla = np.zeros_like(z)
    dlb = None if zb is None else np.zeros((B, L, gh, dv), dtype=np.float64)
    ds0 = np.zeros((B, H, dk, dv), dtype=np.float64)
    rc = _load().oracle_gla_bwd_ext(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(zz), gh, float(inv_tau), _ptr(s0),
                                    _ptr(dO), _ptr(dsf), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dla), _ptr(dlb),
                                    _ptr(ds0), B, H, L, dk, dv, Hg, Wg, int(mode))
    if rc:
        raise ValueError("oracle_gla_bwd_ext rejected the arguments (rc=%d)" % rc)
    return dq, dkk, dvv, dla, dlb, ds0


def gla_bwd(q, k, v, z, inv_tau, dO, grid_h, grid_w, mode):
    """(dq, dk, dv, dlogalpha) of sum(o * dO); dlogalpha is shaped like z."""
    q, k, v, z, dO = _f64(q), _f64(k), _f64(v), _f64(z), _f64(dO)
    B, L, H, dk = q.shape
    dv = v.shape[3]
    gh = z.shape[2]
    dq = np.zeros_like(q)
    dkk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    dla = np.zeros_like(z)
    rc = _load().oracle_gla_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(z), gh, float(inv_tau), _ptr(dO),
                                _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dla),
                                B, H, L, dk, dv, grid_h, grid_w, int(mode))
    if rc:
        raise ValueError("oracle_gla_bwd rejected the arguments (rc=%d)" % rc)
    return dq, dkk, dvv, dla


def epilogue(o, r, gamma=None, eps=1e-5):
    """y = Swish(r) * RMSNorm_dv(o) * gamma over the last axis."""
    o, r = _f64(o), _f64(r)
    dv = o.shape[-1]
    rows = o.size // dv if dv else 0
    g = None if gamma is None else _f64(gamma)
    y = np.zeros_like(o)
    rc = _load().oracle_epilogue(_ptr(o), _ptr(r), _ptr(g), float(eps), _ptr(y), rows, dv)
    if rc:
        raise ValueError("oracle_epilogue rejected the arguments")
    return y


def epilogue_bwd(o, r, dy, gamma=None, eps=1e-5):
    """Gradients (d_o, d_r, d_gamma) of sum(dy * epilogue(o, r, gamma, eps))."""
    o, r, dy = _f64(o), _f64(r), _f64(dy)
    dv = o.shape[-1]
    rows = o.size // dv if dv else 0
    g = None if gamma is None else _f64(gamma)
    d_o, d_r = np.zeros_like(o), np.zeros_like(o)
    d_gamma = np.zeros(dv, dtype=np.float64)
    rc = _load().oracle_epilogue_bwd(_ptr(o), _ptr(r), _ptr(g), float(eps), _ptr(dy), _ptr(d_o), _ptr(d_r),
                                     _ptr(d_gamma), rows, dv)
    if rc:
        raise ValueError("oracle_epilogue_bwd rejected the arguments")
    return d_o, d_r, d_gamma


def srem_dwconv_bwd(x, w, dy, mode):
    """Gradients (dx [B,Hg,Wg,C] grid order, dw [C,3,3], dbias [C]) of sum(dy * srem_dwconv(x, w, bias, mode))
    for dy [B,L,C] in scan order."""
    x, w, dy = _f64(x), _f64(w), _f64(dy)
    B, Hg, Wg, C = x.shape
    dx = np.zeros_like(x)
    dw = np.zeros((C, 3, 3), dtype=np.float64)
    db = np.zeros(C, dtype=np.float64)
    rc = _load().oracle_srem_dwconv_bwd(_ptr(x), _ptr(w), _ptr(dy), _ptr(dx), _ptr(dw), _ptr(db),
                                        B, Hg, Wg, C, int(mode))
    if rc:
        raise ValueError("oracle_srem_dwconv_bwd rejected the arguments (rc=%d)" % rc)
    return dx, dw, db


def gate_proj_fwd(x, W1, W2, b=None):
    """z = (x W1) W2 + b over the last axis of x [..., D]; returns (z [..., dk], u = x W1 [..., R])."""
    x, W1, W2 = _f64(x), _f64(W1), _f64(W2)
    D, R, dk = W1.shape[0], W1.shape[1], W2.shape[1]
    rows = x.size // D
    bb = None if b is None else _f64(b)
    z = np.zeros(x.shape[:-1] + (dk,), dtype=np.float64)
    u = np.zeros(x.shape[:-1] + (R,), dtype=np.float64)
    rc = _load().oracle_gate_proj_fwd(_ptr(x), _ptr(W1), _ptr(W2), _ptr(bb), _ptr(z), _ptr(u), rows, D, R, dk)
    if rc:
        raise ValueError("oracle_gate_proj_fwd rejected the arguments")
    return z, u


def gate_proj_bwd(x, W1, W2, z, dlog_alpha, inv_tau):
    """Gradients (dx, dW1, dW2, db) of sum(dlog_alpha * inv_tau * logsigmoid(z)) for z = gate_proj_fwd(x, W1, W2, b)."""
    x, W1, W2, z, dla = _f64(x), _f64(W1), _f64(W2), _f64(z), _f64(dlog_alpha)
    D, R, dk = W1.shape[0], W1.shape[1], W2.shape[1]
    rows = x.size // D
    dx = np.zeros_like(x)
    dW1, dW2, db = np.zeros((D, R)), np.zeros((R, dk)), np.zeros(dk)
    rc = _load().oracle_gate_proj_bwd(_ptr(x), _ptr(W1), _ptr(W2), _ptr(z), _ptr(dla), float(inv_tau), _ptr(dx),
                                      _ptr(dW1), _ptr(dW2), _ptr(db), rows, D, R, dk)
    if rc:
        raise ValueError("oracle_gate_proj_bwd rejected the arguments (rc=%d)" % rc)
    return dx, dW1, dW2, db


def srem_dwconv(x, w, bias, mode):
    """x [B,Hg,Wg,C] grid order; w [C,3,3]; bias [C] or None -> y [B,L,C] in scan order."""
    x, w = _f64(x), _f64(w)
    B, Hg, Wg, C = x.shape
    bb = None if bias is None else _f64(bias)
    y = np.zeros((B, Hg * Wg, C), dtype=np.float64)
    rc = _load().oracle_srem_dwconv(_ptr(x), _ptr(w), _ptr(bb), _ptr(y), B, Hg, Wg, C, int(mode))
    if rc:
        raise ValueError("oracle_srem_dwconv rejected the arguments")
    return y

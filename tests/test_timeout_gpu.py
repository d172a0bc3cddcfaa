"""Bounded device waits: expiry is reported, nothing is left in flight, the context survives.

Every kernel wait on a completion barrier is bounded.  The environment variable
DIG_DEVICE_WAIT_LIMIT_NS (read on every call; a test hook) shortens the bound;
at 1 ns each kernel's first wait on a copy or a product gives up.  The call must
then still return, the device status must read DIG_ERR_DEVICE_TIMEOUT, the
stream must synchronize without a CUDA error (no trap, no fault: each CTA drains
its copies and products before it releases TMEM and exits), and the next call
with the normal bound must be correct.  Covered: the tile-copy kernels (bf16,
d_k = 32, d_v = 64) and the exact kernels (fp32 inputs; bf16 with d_k = 36,
d_v = 72), forward, full backward and the backward from a forward's records.
"""
import contextlib
import os

import pytest
import torch

import oracle
from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import dev, host, rel_err, tol

pytestmark = pytest.mark.gpu

CASES = [  # (dtype, d_k, d_v, grid_h, grid_w)
    ("bf16", 32, 64, 16, 32),   # tile-copy kernels: 512 tokens, 4 chunks per sequence
    ("f32", 64, 64, 16, 24),    # exact kernels, 64-token chunks
    ("bf16", 36, 72, 16, 24),   # exact kernels, 128-token forward / 64-token backward chunks
]


def _dig():
    from gated_linear_attention_fwd_b200 import dig
    return dig


@contextlib.contextmanager
def wait_bound_ns(v):
    old = os.environ.get("DIG_DEVICE_WAIT_LIMIT_NS")
    os.environ["DIG_DEVICE_WAIT_LIMIT_NS"] = str(v)
    try:
        yield
    finally:
        if old is None:
            del os.environ["DIG_DEVICE_WAIT_LIMIT_NS"]
        else:
            os.environ["DIG_DEVICE_WAIT_LIMIT_NS"] = old


def _problem(case):
    dtype, dk, dv, gh, gw = case
    w = inputs.custom(2, 3, gh, gw, dk, dv, dtype=dtype)
    x = inputs.make_inputs(w, seed=77 + dk)
    t = {n: dev(x[n], dtype) for n in ("q", "k", "v", "dO")}
    t["z"] = dev(x["z"])
    return w, x, t


def _fwd(w, t, mode):
    dig = _dig()
    o = torch.full((w.B, w.L, w.H, w.dv), float("nan"), device="cuda")
    ws = dig.new_workspace(w.B, w.H, w.L, w.dk, w.dv)
    dig.dig_gla_fwd(t["q"], t["k"], t["v"], t["z"], w.inv_tau, o, w.grid_h, w.grid_w, mode, ws)
    return o, ws


def _bwd(w, t, mode, fws=None):
    dig = _dig()
    g = [torch.full_like(t["q"], float("nan"), dtype=torch.float32),
         torch.full_like(t["k"], float("nan"), dtype=torch.float32),
         torch.full_like(t["v"], float("nan"), dtype=torch.float32),
         torch.full_like(t["z"], float("nan"))]
    ws = dig.new_workspace(w.B, w.H, w.L, w.dk, w.dv, backward=True)
    if fws is None:
        dig.dig_gla_bwd(t["q"], t["k"], t["v"], t["z"], w.inv_tau, t["dO"], *g, w.grid_h, w.grid_w, mode, ws)
    else:
        dig.dig_gla_bwd_saved(t["q"], t["k"], t["v"], t["z"], w.inv_tau, t["dO"], *g, w.grid_h, w.grid_w, mode,
                              fws, ws)
    return g, ws


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("mode", [0, 3])
def test_forward_wait_expiry_is_reported_and_the_context_survives(case, mode):
    dig = _dig()
    w, x, t = _problem(case)
    with wait_bound_ns(1):
        _, ws = _fwd(w, t, mode)
        torch.cuda.synchronize()  # no CUDA error: the CTAs drained and exited
    assert dig.dig_read_status(ws) == dig.DIG_ERR_DEVICE_TIMEOUT
    o, ws = _fwd(w, t, mode)
    assert dig.dig_read_status(ws) == dig.DIG_OK
    ref = oracle.gla_fwd(x["q"], x["k"], x["v"], x["z"], w.inv_tau, w.grid_h, w.grid_w, mode)
    assert rel_err(host(o), ref) <= tol(w.dtype)


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("saved", [False, True])
def test_backward_wait_expiry_is_reported_and_the_context_survives(case, saved):
    dig = _dig()
    w, x, t = _problem(case)
    mode = 1
    fws = _fwd(w, t, mode)[1] if saved else None
    if saved and dig.dig_read_status(fws) != dig.DIG_OK:
        pytest.fail("forward status %d" % dig.dig_read_status(fws))
    with wait_bound_ns(1):
        _, ws = _bwd(w, t, mode, fws)
        torch.cuda.synchronize()
    assert dig.dig_read_status(ws) == dig.DIG_ERR_DEVICE_TIMEOUT
    g, ws = _bwd(w, t, mode, fws)
    assert dig.dig_read_status(ws) == dig.DIG_OK
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], x["z"], w.inv_tau, x["dO"], w.grid_h, w.grid_w, mode)
    errs = [rel_err(host(a), r) for a, r in zip(g, ref)]
    assert max(errs) <= tol(w.dtype), errs

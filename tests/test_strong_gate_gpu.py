"""Strong gates: chunks whose decay leaves the range of the chunk factorisation
(more than 115 halvings over half a chunk) are recomputed exactly by
gla_strong.cu instead of being refused.  GPU parity against the fp64 oracle for
the forward (o, and y with the epilogue), the backward and the backward from the
forward's records, on gates with alpha = 0 to fp32 precision, on tau = 1 gates
with z ~ N(-3, 1), and on a mix of flagged and ordinary chunks; every scan order.

Acceptance as in the other parity tests: max|d| / rms(oracle) <= 1e-4 for fp32
inputs, <= 1e-2 for bf16 inputs.  d log alpha is normalised by the larger of
its own rms and the rms of its per-token terms sum_h q * dq (with alpha = 0 the
exact d log alpha is zero: its terms cancel, q dq = k dk token by token).
"""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import dev, host, rel_err, tol

pytestmark = pytest.mark.gpu


def _dig():
    from gated_linear_attention_fwd_b200 import dig
    return dig


CASES = [
    # (B, H, grid_h, grid_w, dk, dv, dtype, gate_heads, inv_tau, kind)
    (1, 2, 16, 16, 32, 64, "bf16", 1, 1.0, "alpha0"),
    (1, 2, 16, 24, 32, 64, "f32", 1, 1.0, "alpha0"),
    (2, 3, 16, 16, 32, 64, "bf16", 1, 1.0, "tau1"),
    (1, 2, 20, 20, 36, 72, "f32", 1, 1.0, "tau1"),
    (2, 2, 32, 32, 32, 64, "bf16", 1, 1 / 16, "mixed"),
    (1, 2, 24, 32, 64, 64, "bf16", 2, 1 / 16, "mixed"),   # one gate per head
    (1, 1, 10, 13, 32, 64, "bf16", 1, 1.0, "mixed"),      # ragged: 130 tokens
    (1, 2, 16, 24, 36, 72, "f32", 1, 1 / 16, "mixed"),
    (1, 2, 24, 24, 36, 72, "bf16", 1, 1 / 16, "mixed"),
]


def _setup(case):
    B, H, Hg, Wg, dk, dv, dtype, gh, inv_tau, kind = case
    w = inputs.custom(B, H, Hg, Wg, dk, dv, dtype=dtype, inv_tau=inv_tau)
    x = inputs.make_inputs(w, seed=7000 + Hg * Wg + dk, with_epilogue=True)
    z = inputs.strong_gate(w, kind, seed=8000 + Hg, gate_heads=gh)
    return w, x, z


def _dla_err(got, ref, q, dq, gh):
    """max|d| / max(rms(ref), rms(sum over the heads of a gate of q * dq))."""
    B, L, H, dk = q.shape
    terms = (q * dq).reshape(B, L, gh, H // gh, dk).sum(axis=3)
    scale = max(np.sqrt(np.mean(ref * ref)), np.sqrt(np.mean(terms * terms)))
    return float(np.max(np.abs(got - ref)) / scale)


@pytest.mark.parametrize("mode", range(4))
@pytest.mark.parametrize("case", CASES)
def test_strong_gates_forward(case, mode):
    dig = _dig()
    w, x, z = _setup(case)
    B, L, H, dk, dv = w.B, w.L, w.H, w.dk, w.dv
    q, k, v, r = (dev(x[n], w.dtype) for n in ("q", "k", "v", "r"))
    zz = dev(z)
    gamma = dev(1.0 + 0.1 * np.random.default_rng(5).standard_normal(dv))
    o = torch.full((B, L, H, dv), float("nan"), device="cuda")
    y = torch.full_like(o, float("nan"))
    ws = dig.new_workspace(B, H, L, dk, dv, gate_heads=z.shape[2])
    dig.dig_gla_fwd(q, k, v, zz, w.inv_tau, o, w.grid_h, w.grid_w, mode, ws, r=r, gamma=gamma, eps=1e-5, y=y)
    assert dig.dig_read_status(ws) == 0
    ref = oracle.gla_fwd(x["q"], x["k"], x["v"], z, w.inv_tau, w.grid_h, w.grid_w, mode)
    assert rel_err(host(o), ref) <= tol(w.dtype), rel_err(host(o), ref)
    yref = oracle.epilogue(ref, x["r"], host(gamma), eps=1e-5)
    assert rel_err(host(y), yref) <= tol(w.dtype), rel_err(host(y), yref)
    if case[-1] == "alpha0":  # the closed form: only the current token survives
        qk = np.einsum("blhc,blhc->blh", x["q"].astype(np.float64), x["k"].astype(np.float64))
        closed = qk[..., None] * x["v"].astype(np.float64)
        assert rel_err(host(o), closed) <= tol(w.dtype)


@pytest.mark.parametrize("saved", [False, True])
@pytest.mark.parametrize("mode", range(4))
@pytest.mark.parametrize("case", CASES)
def test_strong_gates_backward(case, mode, saved):
    dig = _dig()
    w, x, z = _setup(case)
    B, L, H, dk, dv = w.B, w.L, w.H, w.dk, w.dv
    gh = z.shape[2]
    q, k, v, dO = (dev(x[n], w.dtype) for n in ("q", "k", "v", "dO"))
    zz = dev(z)
    dq = torch.full((B, L, H, dk), float("nan"), device="cuda")
    dkk, dvv = torch.full_like(dq, float("nan")), torch.full((B, L, H, dv), float("nan"), device="cuda")
    dla = torch.full(tuple(zz.shape), float("nan"), device="cuda")
    ws = dig.new_workspace(B, H, L, dk, dv, backward=True, gate_heads=gh)
    if saved:
        fws = dig.new_workspace(B, H, L, dk, dv, gate_heads=gh)
        o = torch.empty(B, L, H, dv, device="cuda")
        dig.dig_gla_fwd(q, k, v, zz, w.inv_tau, o, w.grid_h, w.grid_w, mode, fws)
        assert dig.dig_read_status(fws) == 0
        dig.dig_gla_bwd_saved(q, k, v, zz, w.inv_tau, dO, dq, dkk, dvv, dla, w.grid_h, w.grid_w, mode, fws, ws)
    else:
        dig.dig_gla_bwd(q, k, v, zz, w.inv_tau, dO, dq, dkk, dvv, dla, w.grid_h, w.grid_w, mode, ws)
    assert dig.dig_read_status(ws) == 0
    rq, rk, rv, rla = oracle.gla_bwd(x["q"], x["k"], x["v"], z, w.inv_tau, x["dO"], w.grid_h, w.grid_w, mode)
    errs = {"dq": rel_err(host(dq), rq), "dk": rel_err(host(dkk), rk), "dv": rel_err(host(dvv), rv),
            "dlogalpha": _dla_err(host(dla), rla, x["q"].astype(np.float64), rq, gh)}
    assert max(errs.values()) <= tol(w.dtype), errs


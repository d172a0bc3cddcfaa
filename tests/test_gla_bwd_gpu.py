"""GPU parity of dig_gla_bwd (through the C ABI) against the fp64 oracle.

Acceptance: max|d| / rms(oracle) <= 1e-4 for fp32 inputs, <= 1e-2 for bf16
inputs, for each of dq, dk, dv and dlog(alpha).  dq/dk/dv stored as bf16 must be
exactly the round-to-nearest-even of the same kernel's fp32 result.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import dev, host, oracle_bwd, rel_err, tol, workload_inputs

pytestmark = pytest.mark.gpu


def _dig():
    from gated_linear_attention_fwd_b200 import dig
    return dig


def run_bwd(w, x, mode, out_dtype="f32", gate=None, ws=None):
    dig = _dig()
    B, L, H, dk, dv = w.B, w.L, w.H, w.dk, w.dv
    q, k, v, dO = dev(x["q"], w.dtype), dev(x["k"], w.dtype), dev(x["v"], w.dtype), dev(x["dO"], w.dtype)
    zz = gate if gate is not None else x["z"]
    z = dev(zz)
    odt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    dq = torch.full((B, L, H, dk), float("nan"), dtype=odt, device="cuda")
    dkk = torch.full_like(dq, float("nan"))
    dvv = torch.full((B, L, H, dv), float("nan"), dtype=odt, device="cuda")
    dla = torch.full(tuple(z.shape), float("nan"), dtype=torch.float32, device="cuda")
    if ws is None:
        ws = dig.new_workspace(B, H, L, dk, dv, backward=True, gate_heads=z.shape[2])
    dig.dig_gla_bwd(q, k, v, z, w.inv_tau, dO, dq, dkk, dvv, dla, w.grid_h, w.grid_w, mode, ws)
    st = dig.dig_read_status(ws)
    return (dq, dkk, dvv, dla), st


def _check(got, ref, dtype):
    errs = [rel_err(host(g), r) for g, r in zip(got, ref)]
    assert max(errs) <= tol(dtype), dict(zip(("dq", "dk", "dv", "dlogalpha"), errs))


@pytest.mark.parametrize("index", range(len(inputs.WORKLOADS)))
@pytest.mark.parametrize("mode", range(4))
def test_bwd_matches_oracle_on_every_workload(index, mode):
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    got, st = run_bwd(w, x, mode, "f32")
    assert st == 0
    _check(got, oracle_bwd(index, mode), w.dtype)


@pytest.mark.parametrize("index", [2, 4])
def test_bwd_bf16_outputs_are_rounded_fp32_outputs(index):
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    g32, _ = run_bwd(w, x, 3, "f32")
    g16, st = run_bwd(w, x, 3, "bf16")
    assert st == 0
    for a, b in zip(g16[:3], g32[:3]):
        assert torch.equal(a, b.to(torch.bfloat16))


EDGE = [
    # (B, H, grid_h, grid_w, dk, dv, dtype, gate_heads, inv_tau, zshift)
    (1, 2, 10, 13, 32, 64, "bf16", 1, 1 / 16, 0.0),     # ragged: 130 tokens
    (2, 1, 1, 5, 36, 72, "bf16", 1, 1 / 16, 0.0),       # shorter than one chunk
    (1, 1, 3, 37, 64, 64, "f32", 1, 1 / 16, 0.0),       # fp32 ragged
    (3, 4, 16, 40, 32, 64, "bf16", 4, 1 / 16, 0.0),     # one gate per head
    (2, 3, 20, 33, 36, 72, "bf16", 3, 1.0, 1.0),        # tau = 1 gates
    (64, 6, 16, 16, 32, 64, "bf16", 1, 1 / 16, 0.0),    # 384 short sequences: more units than CTAs
    (1, 1, 64, 64, 32, 64, "bf16", 1, 1 / 16, 0.0),     # one sequence of many chunks over the scan ranges
    (1, 1, 128, 160, 32, 64, "bf16", 1, 1 / 16, 0.0),   # 160 chunks: two load windows per scan range
    (1, 1, 2, 2, 32, 64, "f32", 1, 1 / 16, 0.0),        # 4 tokens
    (1, 2, 16, 24, 36, 72, "f32", 1, 1 / 16, 0.0),     # fp32 d_v = 72 > the 64-token chunk
]


@pytest.mark.parametrize("case", EDGE)
@pytest.mark.parametrize("mode", [0, 3])
def test_bwd_edge_cases(case, mode):
    B, H, Hg, Wg, dk, dv, dtype, gh, inv_tau, zshift = case
    w = inputs.custom(B, H, Hg, Wg, dk, dv, dtype=dtype, inv_tau=inv_tau)
    x = inputs.make_inputs(w, seed=4321 + Hg * Wg)
    z = np.ascontiguousarray(np.repeat(x["z"], gh, axis=2) + zshift, dtype=np.float32)
    if gh > 1:
        z = z + np.random.default_rng(4).standard_normal(z.shape).astype(np.float32)
    got, st = run_bwd(w, x, mode, "f32", gate=z)
    assert st == 0
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], z, inv_tau, x["dO"], Hg, Wg, mode)
    _check(got, ref, dtype)


def test_bwd_workspace_is_reusable_across_calls():
    w = inputs.WORKLOADS[2]
    x = workload_inputs(2)
    dig = _dig()
    ws = dig.new_workspace(w.B, w.H, w.L, w.dk, w.dv, backward=True)
    a, _ = run_bwd(w, x, 2, "f32", ws=ws)
    b, st = run_bwd(w, x, 2, "f32", ws=ws)
    assert st == 0
    for u, v in zip(a[:3], b[:3]):
        assert torch.equal(u, v)
    assert rel_err(host(a[3]), host(b[3])) < 1e-5   # dlog(alpha) sums heads with atomics (fp32 order)


def run_bwd_saved(w, x, mode, out_dtype="f32", gate=None):
    """dig_gla_fwd, then dig_gla_bwd_saved on the forward's workspace."""
    dig = _dig()
    B, L, H, dk, dv = w.B, w.L, w.H, w.dk, w.dv
    q, k, v, dO = dev(x["q"], w.dtype), dev(x["k"], w.dtype), dev(x["v"], w.dtype), dev(x["dO"], w.dtype)
    z = dev(gate if gate is not None else x["z"])
    gh = z.shape[2]
    o = torch.empty(B, L, H, dv, dtype=torch.float32, device="cuda")
    fws = dig.new_workspace(B, H, L, dk, dv, gate_heads=gh)
    dig.dig_gla_fwd(q, k, v, z, w.inv_tau, o, w.grid_h, w.grid_w, mode, fws)
    odt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    dq = torch.full((B, L, H, dk), float("nan"), dtype=odt, device="cuda")
    dkk = torch.full_like(dq, float("nan"))
    dvv = torch.full((B, L, H, dv), float("nan"), dtype=odt, device="cuda")
    dla = torch.full(tuple(z.shape), float("nan"), dtype=torch.float32, device="cuda")
    ws = dig.new_workspace(B, H, L, dk, dv, backward=True, gate_heads=gh)
    dig.dig_gla_bwd_saved(q, k, v, z, w.inv_tau, dO, dq, dkk, dvv, dla, w.grid_h, w.grid_w, mode, fws, ws)
    st = dig.dig_read_status(ws)
    assert dig.dig_read_status(fws) == 0
    return (dq, dkk, dvv, dla), st


@pytest.mark.parametrize("index", range(len(inputs.WORKLOADS)))
@pytest.mark.parametrize("mode", range(4))
def test_bwd_saved_matches_oracle_on_every_workload(index, mode):
    """The backward on the forward's gate factors and chunk states (workload 4's
    backward uses shorter chunks than its forward, so it takes the full backward)."""
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    got, st = run_bwd_saved(w, x, mode, "f32")
    assert st == 0
    _check(got, oracle_bwd(index, mode), w.dtype)


@pytest.mark.parametrize("case", EDGE)
def test_bwd_saved_edge_cases(case):
    B, H, Hg, Wg, dk, dv, dtype, gh, inv_tau, zshift = case
    w = inputs.custom(B, H, Hg, Wg, dk, dv, dtype=dtype, inv_tau=inv_tau)
    x = inputs.make_inputs(w, seed=4321 + Hg * Wg)
    z = np.ascontiguousarray(np.repeat(x["z"], gh, axis=2) + zshift, dtype=np.float32)
    if gh > 1:
        z = z + np.random.default_rng(4).standard_normal(z.shape).astype(np.float32)
    got, st = run_bwd_saved(w, x, 1, "f32", gate=z)
    assert st == 0
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], z, inv_tau, x["dO"], Hg, Wg, 1)
    _check(got, ref, dtype)


def test_bwd_saved_agrees_with_the_full_backward():
    w = inputs.WORKLOADS[2]
    x = workload_inputs(2)
    a, _ = run_bwd(w, x, 2, "f32")
    b, st = run_bwd_saved(w, x, 2, "f32")
    assert st == 0
    for u, v in zip(a, b):
        assert rel_err(host(v), host(u)) < 1e-4

"""GPU parity of dig_gla_fwd (called through the C ABI) against the fp64 oracle.

Acceptance: max|d| / rms(oracle) <= 1e-4 for fp32 inputs, <= 1e-2 for bf16
inputs (fp32 accumulation).  Outputs stored as bf16 are checked to be exactly
the round-to-nearest-even of the same kernel's fp32 result.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import dev, host, oracle_fwd, rel_err, tol, workload_inputs

pytestmark = pytest.mark.gpu


def _dig():
    from gated_linear_attention_fwd_b200 import dig
    return dig


def run_fwd(w, x, mode, out_dtype="f32", epilogue=False, gamma=None, ws=None, gate=None):
    dig = _dig()
    B, L, H, dk, dv = w.B, w.L, w.H, w.dk, w.dv
    q, k, v = dev(x["q"], w.dtype), dev(x["k"], w.dtype), dev(x["v"], w.dtype)
    z = dev(gate if gate is not None else x["z"])
    odt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    o = torch.full((B, L, H, dv), float("nan"), dtype=odt, device="cuda")
    r = y = g = None
    if epilogue:
        r = dev(x["r"], w.dtype)
        y = torch.full_like(o, float("nan"))
        if gamma is not None:
            g = dev(gamma)
    if ws is None:
        ws = dig.new_workspace(B, H, L, dk, dv, gate_heads=z.shape[2])
    dig.dig_gla_fwd(q, k, v, z, w.inv_tau, o, w.grid_h, w.grid_w, mode, ws, r=r, gamma=g, eps=1e-5, y=y)
    st = dig.dig_read_status(ws)
    return o, y, st


@pytest.mark.parametrize("index", range(len(inputs.WORKLOADS)))
@pytest.mark.parametrize("mode", range(4))
def test_fwd_matches_oracle_on_every_workload(index, mode):
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    o, _, st = run_fwd(w, x, mode, "f32")
    assert st == 0
    err = rel_err(host(o), oracle_fwd(index, mode))
    assert err <= tol(w.dtype), err


@pytest.mark.parametrize("index", [1, 2, 4])
def test_bf16_output_is_rounded_fp32_output(index):
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    o32, _, _ = run_fwd(w, x, 2, "f32")
    o16, _, st = run_fwd(w, x, 2, "bf16")
    assert st == 0
    assert torch.equal(o16, o32.to(torch.bfloat16))


def test_fwd_epilogue_matches_oracle():
    index = 3  # DiG-S/2 at 1792^2 carries the Swish(r) * RMSNorm(o) epilogue
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    rng = np.random.default_rng(5)
    gamma = (1.0 + 0.1 * rng.standard_normal(w.dv)).astype(np.float32)
    for mode in range(4):
        o, y, st = run_fwd(w, x, mode, "f32", epilogue=True, gamma=gamma)
        assert st == 0
        o_ref = oracle_fwd(index, mode)
        y_ref = oracle.epilogue(o_ref, x["r"], gamma, eps=1e-5)
        assert rel_err(host(o), o_ref) <= 1e-2
        assert rel_err(host(y), y_ref) <= 1e-2
    o16, y16, _ = run_fwd(w, x, 1, "bf16", epilogue=True, gamma=gamma)
    o32, y32, _ = run_fwd(w, x, 1, "f32", epilogue=True, gamma=gamma)
    assert torch.equal(y16, y32.to(torch.bfloat16))


@pytest.mark.parametrize("mode", [1, 2, 3])
@pytest.mark.parametrize("index", [0, 2, 4])
def test_scan_mode_equals_row_scan_of_reoriented_input_bitexact(index, mode):
    """gla(mode m, x) == reorient^-1(gla(row-forward, reorient(x))): the fused
    permutation changes only which rows are read and written.  Bit for bit where
    the same kernels see the chunk's tokens in scan order.  On workload 2 (bf16,
    d_k = 32, d_v = 64) the row-forward call runs the tile-copy kernels, which
    hold the reversed orders' tiles in grid order (the products that sum over
    tokens add the same terms in the opposite order), and the column orders'
    outputs come from the exact kernel; there the two agree to fp32 accumulation
    rounding instead (bounded here by the fp32-input tolerance, far below the O(1)
    error of a wrong permutation)."""
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    perm = oracle.scan_index(mode, w.grid_h, w.grid_w)
    xp = {k: np.ascontiguousarray(v[:, perm]) for k, v in x.items() if k in ("q", "k", "v", "z")}
    o_m, _, _ = run_fwd(w, x, mode, "f32")
    o_r, _, _ = run_fwd(w, xp, 0, "f32")
    o_m = o_m[:, torch.as_tensor(perm, device="cuda")]
    if index == 2:
        assert rel_err(host(o_m), host(o_r)) <= 1e-4
    else:
        assert torch.equal(o_m, o_r)


EDGE = [
    # (B, H, grid_h, grid_w, dk, dv, dtype, gate_heads, inv_tau, zshift)
    (1, 2, 10, 13, 32, 64, "bf16", 1, 1 / 16, 0.0),     # ragged: 130 tokens = 128 + 2
    (2, 1, 1, 5, 36, 72, "bf16", 1, 1 / 16, 0.0),       # shorter than one chunk
    (1, 1, 3, 37, 64, 64, "f32", 1, 1 / 16, 0.0),       # fp32 ragged: 111 = 64 + 47
    (3, 4, 16, 40, 32, 64, "bf16", 4, 1 / 16, 0.0),     # one gate per head
    (2, 3, 20, 33, 36, 72, "bf16", 3, 1.0, 1.0),        # tau = 1 gates (alpha ~ sigmoid(N(1, 1.4)))
    (64, 6, 16, 16, 32, 64, "bf16", 1, 1 / 16, 0.0),    # 384 two-chunk sequences: more units than CTAs
    (1, 1, 64, 64, 32, 64, "bf16", 1, 1 / 16, 0.0),     # one sequence of 32 chunks over the 16 scan ranges
    (1, 1, 128, 160, 32, 64, "bf16", 1, 1 / 16, 0.0),   # 160 chunks: two load windows per scan range
    (1, 1, 2, 2, 32, 64, "f32", 1, 1 / 16, 0.0),        # 4 tokens
    (1, 2, 16, 24, 36, 72, "f32", 1, 1 / 16, 0.0),     # fp32 d_v = 72 > the 64-token chunk
]


@pytest.mark.parametrize("case", EDGE)
@pytest.mark.parametrize("mode", [0, 3])
def test_fwd_edge_cases(case, mode):
    B, H, Hg, Wg, dk, dv, dtype, gh, inv_tau, zshift = case
    w = inputs.custom(B, H, Hg, Wg, dk, dv, dtype=dtype, inv_tau=inv_tau)
    x = inputs.make_inputs(w, seed=1234 + Hg * Wg)
    z = np.ascontiguousarray(np.repeat(x["z"], gh, axis=2) + zshift, dtype=np.float32)
    if gh > 1:
        z = z + np.random.default_rng(3).standard_normal(z.shape).astype(np.float32)
    o, _, st = run_fwd(w, x, mode, "f32", gate=z)
    assert st == 0
    ref = oracle.gla_fwd(x["q"], x["k"], x["v"], z, inv_tau, Hg, Wg, mode)
    err = rel_err(host(o), ref)
    assert err <= tol(dtype), err


def test_workspace_is_reusable_across_calls():
    w = inputs.WORKLOADS[2]
    x = workload_inputs(2)
    dig = _dig()
    ws = dig.new_workspace(w.B, w.H, w.L, w.dk, w.dv)
    a, _, _ = run_fwd(w, x, 1, "f32", ws=ws)
    b, _, _ = run_fwd(w, x, 1, "f32", ws=ws)
    c, _, st = run_fwd(w, x, 1, "f32", ws=ws)
    assert st == 0 and torch.equal(a, b) and torch.equal(b, c)


@pytest.mark.parametrize("which", ["key", "value"])
def test_ext_gate_out_of_range_is_reported_not_faulted(which):
    """dig_gla_fwd computes strong key gates (tests/test_strong_gate_gpu.py); the
    extended entry point has no strong-gate path and reports such a chunk in the
    status word instead, for its key gate and for its value gate alike."""
    dig = _dig()
    w = inputs.custom(1, 1, 16, 16, 32, 64, dtype="f32", inv_tau=1.0)
    x = inputs.make_inputs(w, seed=99)
    strong = np.full_like(x["z"], -300.0)   # alpha = e^-300 per token: far outside the factorisation's range
    z = strong if which == "key" else x["z"]
    zb = np.full((w.B, w.L, 1, w.dv), -300.0 if which == "value" else 0.0, dtype=np.float32)
    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    o = torch.empty(w.B, w.L, w.H, w.dv, device="cuda")
    ws = dig.new_ext_workspace(w.B, w.H, w.L, w.dk, w.dv, dtype=torch.float32)
    dig.dig_gla_fwd_ext(q, k, v, dev(z), w.inv_tau, o, w.grid_h, w.grid_w, 0, ws, zb=dev(zb))
    assert dig.dig_read_status(ws) == dig.DIG_ERR_GATE_RANGE

"""GPU parity of the extended entry points (value gate beta, state input / output)
against the fp64 oracle's gla_fwd_ext / gla_bwd_ext, called through the C ABI.

The extended calls run the fp32 kernels (bf16 inputs are widened exactly), so
the acceptance bound is the fp32 one, max|d| / rms(oracle) <= 1e-4, for o,
S_final, dq, dk, dv, dlog(alpha), dlog(beta) and dS0.  Value-gate logits are
N(0, 1) (beta = sigmoid(zb)^(1/tau) spread over (0.8, 1) at tau = 16), the
initial state and the final-state gradient N(0, 1) / sqrt(d_k).
"""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import dev, host, rel_err, workload_inputs

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _dig():
    from gated_linear_attention_fwd_b200 import dig
    return dig


def _ext_inputs(w, x, seed, gate_heads=1):
    rng = np.random.default_rng(seed)
    zb = rng.standard_normal((w.B, w.L, gate_heads, w.dv)).astype(np.float32)
    S0 = (rng.standard_normal((w.B, w.H, w.dk, w.dv)) / np.sqrt(w.dk)).astype(np.float32)
    dSf = (rng.standard_normal((w.B, w.H, w.dk, w.dv)) / np.sqrt(w.dk)).astype(np.float32)
    z = x["z"] if gate_heads == 1 else np.ascontiguousarray(
        np.repeat(x["z"], gate_heads, axis=2) + 0.3 * rng.standard_normal((w.B, w.L, gate_heads, w.dk)),
        dtype=np.float32)
    return zb, S0, dSf, z


def run_fwd_ext(w, x, z, zb, S0, mode, grid=None):
    dig = _dig()
    gh, gw = grid or (w.grid_h, w.grid_w)
    B, H, dk, dv = w.B, w.H, w.dk, w.dv
    L = gh * gw
    q, k, v = dev(x["q"], w.dtype), dev(x["k"], w.dtype), dev(x["v"], w.dtype)
    o = torch.full((B, L, H, dv), float("nan"), device="cuda")
    sf = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    ws = dig.new_ext_workspace(B, H, L, dk, dv, dtype=q.dtype, gate_heads=z.shape[2])
    dig.dig_gla_fwd_ext(q, k, v, dev(z), w.inv_tau, o, gh, gw, mode, ws,
                        zb=None if zb is None else dev(zb), S0=None if S0 is None else dev(S0), S_final=sf)
    assert dig.dig_read_status(ws) == dig.DIG_OK
    return o, sf


def run_bwd_ext(w, x, z, zb, S0, dSf, o, mode, grid=None):
    dig = _dig()
    gh, gw = grid or (w.grid_h, w.grid_w)
    B, H, dk, dv = w.B, w.H, w.dk, w.dv
    L = gh * gw
    q, k, v, dO = (dev(x[n], w.dtype) for n in ("q", "k", "v", "dO"))
    gq = torch.full((B, L, H, dk), float("nan"), device="cuda")
    gk = torch.full_like(gq, float("nan"))
    gv = torch.full((B, L, H, dv), float("nan"), device="cuda")
    gla = torch.full((B, L, z.shape[2], dk), float("nan"), device="cuda")
    glb = None if zb is None else torch.full((B, L, z.shape[2], dv), float("nan"), device="cuda")
    gs0 = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    ws = dig.new_ext_workspace(B, H, L, dk, dv, dtype=q.dtype, backward=True, gate_heads=z.shape[2])
    dig.dig_gla_bwd_ext(q, k, v, dev(z), w.inv_tau, dO, gq, gk, gv, gla, gh, gw, mode, ws,
                        zb=None if zb is None else dev(zb), S0=None if S0 is None else dev(S0), o=o,
                        dS_final=None if dSf is None else dev(dSf), dlog_beta=glb, dS0=gs0)
    assert dig.dig_read_status(ws) == dig.DIG_OK
    return gq, gk, gv, gla, glb, gs0


@pytest.mark.parametrize("index", [2, 4])
@pytest.mark.parametrize("mode", range(4))
def test_fwd_ext_matches_oracle(index, mode):
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    zb, S0, _, z = _ext_inputs(w, x, 11 + index)
    o, sf = run_fwd_ext(w, x, z, zb, S0, mode)
    o_ref, sf_ref = oracle.gla_fwd_ext(x["q"], x["k"], x["v"], z, w.inv_tau, w.grid_h, w.grid_w, mode, zb=zb, S0=S0)
    assert rel_err(host(o), o_ref) <= TOL
    assert rel_err(host(sf), sf_ref) <= TOL


@pytest.mark.parametrize("index,mode", [(2, 0), (2, 1), (2, 2), (2, 3), (4, 0), (4, 3)])
def test_bwd_ext_matches_oracle(index, mode):
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    zb, S0, dSf, z = _ext_inputs(w, x, 21 + index)
    o, _ = run_fwd_ext(w, x, z, zb, S0, mode)
    got = run_bwd_ext(w, x, z, zb, S0, dSf, o, mode)
    ref = oracle.gla_bwd_ext(x["q"], x["k"], x["v"], z, w.inv_tau, x["dO"], w.grid_h, w.grid_w, mode,
                             zb=zb, S0=S0, dSf=dSf)
    errs = {n: rel_err(host(g), r) for n, g, r in zip(("dq", "dk", "dv", "dla", "dlb", "dS0"), got, ref)}
    assert max(errs.values()) <= TOL, errs


EDGE = [
    # (B, H, grid_h, grid_w, dk, dv, dtype, gate_heads)
    (1, 2, 10, 13, 32, 64, "bf16", 1),   # ragged: 130 tokens = 2 chunks of 64 + 2
    (2, 3, 1, 5, 36, 72, "f32", 3),      # shorter than one chunk, one gate per head
    (2, 2, 16, 24, 64, 64, "f32", 2),    # d_k = 64, per-head gates
]


@pytest.mark.parametrize("case", EDGE)
@pytest.mark.parametrize("mode", [0, 3])
def test_ext_edge_cases(case, mode):
    B, H, Hg, Wg, dk, dv, dtype, gh = case
    w = inputs.custom(B, H, Hg, Wg, dk, dv, dtype=dtype)
    x = inputs.make_inputs(w, seed=5150 + Hg * Wg)
    zb, S0, dSf, z = _ext_inputs(w, x, 31 + Hg, gate_heads=gh)
    o, sf = run_fwd_ext(w, x, z, zb, S0, mode)
    o_ref, sf_ref = oracle.gla_fwd_ext(x["q"], x["k"], x["v"], z, w.inv_tau, Hg, Wg, mode, zb=zb, S0=S0)
    assert rel_err(host(o), o_ref) <= TOL
    assert rel_err(host(sf), sf_ref) <= TOL
    got = run_bwd_ext(w, x, z, zb, S0, dSf, o, mode)
    ref = oracle.gla_bwd_ext(x["q"], x["k"], x["v"], z, w.inv_tau, x["dO"], Hg, Wg, mode, zb=zb, S0=S0, dSf=dSf)
    errs = {n: rel_err(host(g), r) for n, g, r in zip(("dq", "dk", "dv", "dla", "dlb", "dS0"), got, ref)}
    assert max(errs.values()) <= TOL, errs


def test_ext_without_beta_or_state_equals_plain_gla():
    """zb, S0 and dS_final absent: the plain recurrence (dig_gla_fwd's and the oracle's gla_fwd / gla_bwd)."""
    index, mode = 2, 1
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    o, sf = run_fwd_ext(w, x, x["z"], None, None, mode)
    assert rel_err(host(o), oracle.gla_fwd(x["q"], x["k"], x["v"], x["z"], w.inv_tau, w.grid_h, w.grid_w,
                                           mode)) <= TOL
    got = run_bwd_ext(w, x, x["z"], None, None, None, None, mode)
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], x["z"], w.inv_tau, x["dO"], w.grid_h, w.grid_w, mode)
    for g, r in zip(got[:4], ref):
        assert rel_err(host(g), r) <= TOL


def test_segment_split_continues_the_state_on_the_gpu():
    """Rows 0..31 then 32..63 of a 64 x 64 grid in row order, the second from the
    first's S_final, equal one call over the whole grid; and the second segment's
    dS0, fed to the first as dS_final, gives the whole call's gradients."""
    w = inputs.custom(2, 3, 64, 64, 32, 64, dtype="bf16")
    x = inputs.make_inputs(w, seed=808)
    zb, S0, dSf, z = _ext_inputs(w, x, 909)
    o, sf = run_fwd_ext(w, x, z, zb, S0, 0)
    half = w.L // 2

    def part(a, sl):
        return np.ascontiguousarray(a[:, sl])

    w_h = inputs.custom(2, 3, 32, 64, 32, 64, dtype="bf16")
    x1 = {n: part(x[n], slice(0, half)) for n in ("q", "k", "v", "dO")}
    x2 = {n: part(x[n], slice(half, None)) for n in ("q", "k", "v", "dO")}
    z1, z2, zb1, zb2 = part(z, slice(0, half)), part(z, slice(half, None)), part(zb, slice(0, half)), \
        part(zb, slice(half, None))
    o1, s1 = run_fwd_ext(w_h, x1, z1, zb1, S0, 0)
    o2, s2 = run_fwd_ext(w_h, x2, z2, zb2, host(s1).astype(np.float32), 0)
    assert rel_err(host(torch.cat([o1, o2], dim=1)), host(o)) <= TOL
    assert rel_err(host(s2), host(sf)) <= TOL
    g = run_bwd_ext(w, x, z, zb, S0, dSf, o, 0)
    g2 = run_bwd_ext(w_h, x2, z2, zb2, host(s1).astype(np.float32), dSf, o2, 0)
    g1 = run_bwd_ext(w_h, x1, z1, zb1, S0, host(g2[5]).astype(np.float32), o1, 0)
    for i in range(5):
        assert rel_err(host(torch.cat([g1[i], g2[i]], dim=1)), host(g[i])) <= TOL, i
    assert rel_err(host(g1[5]), host(g[5])) <= TOL

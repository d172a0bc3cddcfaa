"""GPU parity of the gate projection (dig_gate_proj_fwd / dig_gate_proj_bwd)
against the fp64 oracle, and of the chain gate projection -> GLA forward ->
GLA backward -> gate projection backward.

Bars: fp32 results max|d|/rms(ref) <= 1e-4 (fp32 sums over D <= 1152 products of
exact stored inputs; the weight gradients sum over up to 25088 tokens); bf16 dx
must be the exact round-to-nearest-even of the fp32 dx of the same kernel.  The
chain through the GLA is held to the bf16-input bar of the GLA backward, 1e-2."""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import TORCH, dev, host, rel_err, tol

pytestmark = pytest.mark.gpu


def _fwd_gpu(g, dtype, with_u=True):
    from gated_linear_attention_fwd_b200 import dig
    x = dev(g["x"], dtype)
    D, R = g["W1"].shape
    dk = g["W2"].shape[1]
    rows = x.numel() // D
    z = torch.full((rows, dk), float("nan"), device="cuda")
    u = torch.full((rows, R), float("nan"), device="cuda") if with_u else None
    dig.dig_gate_proj_fwd(x, dev(g["W1"]), dev(g["W2"]), z, dev(g["b"]) if "b" in g else None, u)
    torch.cuda.synchronize()
    return z, u


def _bwd_gpu(g, u, z, dla, inv_tau, dtype, out_dtype):
    from gated_linear_attention_fwd_b200 import dig
    x = dev(g["x"], dtype)
    D, R = g["W1"].shape
    dk = g["W2"].shape[1]
    dx = torch.full(x.shape, float("nan"), dtype=TORCH[out_dtype], device="cuda")
    dW1 = torch.full((D, R), float("nan"), device="cuda")
    dW2 = torch.full((R, dk), float("nan"), device="cuda")
    db = torch.full((dk,), float("nan"), device="cuda")
    dig.dig_gate_proj_bwd(x, dev(g["W1"]), dev(g["W2"]), u, z, dla, inv_tau, dx, dW1, dW2, db)
    torch.cuda.synchronize()
    return dx, dW1, dW2, db


def _check(g, dtype, seed, inv_tau=1.0 / 16.0):
    D = g["W1"].shape[0]
    z, u = _fwd_gpu(g, dtype)
    z_ref, u_ref = oracle.gate_proj_fwd(g["x"], g["W1"], g["W2"], g.get("b"))
    assert rel_err(host(z), z_ref.reshape(-1, z_ref.shape[-1])) <= 1e-4
    assert rel_err(host(u), u_ref.reshape(-1, u_ref.shape[-1])) <= 1e-4
    rng = np.random.default_rng(seed)
    dla = rng.standard_normal(z.shape).astype(np.float32)
    # the backward takes the forward's fp32 z and u as they are
    zh, uh = host(z), host(u)
    dx, dW1, dW2, db = _bwd_gpu(g, u, z, dev(dla), inv_tau, dtype, "f32")
    ref = oracle.gate_proj_bwd(g["x"].reshape(-1, D), g["W1"], g["W2"], zh, dla, inv_tau)
    # dW2 = u^T dz: the oracle recomputes u in fp64; the kernel uses the fp32 u it is given
    assert rel_err(host(dx).reshape(ref[0].shape), ref[0]) <= 1e-4
    assert rel_err(host(dW1), ref[1]) <= 1e-4
    assert rel_err(host(dW2), ref[2]) <= 1e-4
    assert rel_err(host(db), ref[3]) <= 1e-4
    dx16, _, _, _ = _bwd_gpu(g, u, z, dev(dla), inv_tau, dtype, "bf16")
    assert torch.equal(dx16, dx.to(torch.bfloat16))
    return uh


@pytest.mark.parametrize("index", [1, 3, 4])
def test_gate_proj_workloads(index):
    """DiG-S/2 at 256^2 and 1792^2 (384 -> 16 -> 32) and DiG-XL/2 2048^2 (1152 -> 16 -> 36), full size."""
    w = inputs.WORKLOADS[index]
    _check(inputs.gate_proj_inputs(w, 200 + index, with_bias=True), w.dtype, 300 + index)


@pytest.mark.parametrize("rows,D,R,dk", [(1, 8, 16, 32), (65, 24, 5, 6), (130, 16, 20, 3), (64, 384, 32, 128),
                                         (7, 1024, 16, 36),
                                         # bf16: the tensor-core backward (D a multiple of 128 up to 384, R <= 16, d_k <= 32)
                                         (1, 384, 16, 32), (130, 128, 16, 32), (300, 256, 8, 16), (1000, 384, 12, 28)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gate_proj_shapes(rows, D, R, dk, dtype):
    """One token, ragged tiles, ranks padded to 16 and 32, the largest d_k; for bf16 x the
    last four shapes take the tensor-core backward (one and several tiles, 1-3 channel blocks)."""
    rng = np.random.default_rng(rows + D + R + dk)
    x = rng.standard_normal((rows, D))
    g = {"x": inputs.round_bf16(x) if dtype == "bf16" else x.astype(np.float32),
         "W1": (0.1 * rng.standard_normal((D, R))).astype(np.float32),
         "W2": (0.3 * rng.standard_normal((R, dk))).astype(np.float32),
         "b": rng.standard_normal(dk).astype(np.float32)}
    _check(g, dtype, rows)


def test_gate_proj_bwd_zero_rows_clears_gradients():
    from gated_linear_attention_fwd_b200 import dig
    e = torch.empty((0, 16), dtype=torch.bfloat16, device="cuda")
    W1, W2 = torch.ones(16, 4, device="cuda"), torch.ones(4, 8, device="cuda")
    dW1, dW2, db = torch.full((16, 4), 2.0, device="cuda"), torch.full((4, 8), 2.0, device="cuda"), \
        torch.full((8,), 2.0, device="cuda")
    f = torch.empty((0, 8), device="cuda")
    dig.dig_gate_proj_bwd(e, W1, W2, torch.empty((0, 4), device="cuda"), f, f, 0.0625, e.clone(), dW1, dW2, db)
    torch.cuda.synchronize()
    assert torch.all(dW1 == 0) and torch.all(dW2 == 0) and torch.all(db == 0)


def test_gate_chain_through_gla_matches_oracle():
    """x -> z (gate projection) -> GLA forward -> GLA backward (d log alpha) -> dx, dW1, dW2:
    the whole chain on the GPU against the same chain in the oracle."""
    from gated_linear_attention_fwd_b200 import dig
    w = inputs.custom(2, 3, 8, 16, 32, 64, dtype="bf16", gate="lowrank", D=64)
    x = inputs.make_inputs(w, seed=11)
    g = inputs.gate_proj_inputs(w, 12)
    g["W1"] = (g["W1"] * 25.0).astype(np.float32)       # gates away from 1 so d log alpha matters
    B, L, H = w.B, w.L, w.H
    z, u = _fwd_gpu(g, "bf16")
    q, k, v, dO = (dev(x[n], "bf16") for n in ("q", "k", "v", "dO"))
    zz = z.view(B, L, 1, w.dk)
    o = torch.empty(B, L, H, w.dv, device="cuda")
    ws = dig.new_workspace(B, H, L, w.dk, w.dv)
    dig.dig_gla_fwd(q, k, v, zz, w.inv_tau, o, w.grid_h, w.grid_w, 1, ws)
    dq, dk = torch.empty(B, L, H, w.dk, device="cuda"), torch.empty(B, L, H, w.dk, device="cuda")
    dv, dla = torch.empty(B, L, H, w.dv, device="cuda"), torch.empty(B, L, 1, w.dk, device="cuda")
    wsb = dig.new_workspace(B, H, L, w.dk, w.dv, backward=True)
    dig.dig_gla_bwd(q, k, v, zz, w.inv_tau, dO, dq, dk, dv, dla, w.grid_h, w.grid_w, 1, wsb)
    dx, dW1, dW2, db = _bwd_gpu(g, u, z, dla.view(-1, w.dk), w.inv_tau, "bf16", "f32")
    assert dig.dig_read_status(ws) == dig.DIG_OK and dig.dig_read_status(wsb) == dig.DIG_OK
    z_ref, _ = oracle.gate_proj_fwd(g["x"], g["W1"], g["W2"])
    z_ref = z_ref.reshape(B, L, 1, w.dk)
    grads = oracle.gla_bwd(x["q"], x["k"], x["v"], z_ref, w.inv_tau, x["dO"], w.grid_h, w.grid_w, 1)
    ref = oracle.gate_proj_bwd(g["x"].reshape(-1, 64), g["W1"], g["W2"], z_ref.reshape(-1, w.dk),
                               grads[3].reshape(-1, w.dk), w.inv_tau)
    # the chain carries the GLA backward's d log alpha, held to the bf16-input bar
    for got, want in zip((dx, dW1, dW2, db), ref):
        assert rel_err(host(got).reshape(want.shape), want) <= tol("bf16")

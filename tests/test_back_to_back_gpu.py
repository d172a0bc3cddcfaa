"""GPU: ops issued back to back on one stream, sharing their workspaces, with no
synchronisation between them.

Every kernel is launched with programmatic stream serialization, so a kernel may
be scheduled while the one before it is still running.  These calls make the
second forward rewrite the gate factors and chunk states that the first
forward's output kernel and the first backward read, and interleave a conv, so a
write that overtook a read (or a read that overtook a write) shows up as a
parity failure of one of the four results.
"""
import numpy as np
import pytest
import torch

from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import dev, host, oracle_bwd, oracle_fwd, rel_err, tol, workload_inputs

pytestmark = pytest.mark.gpu


def test_back_to_back_forward_and_backward_share_workspaces():
    from gated_linear_attention_fwd_b200 import dig
    index = 2
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    B, L, H, dk, dv = w.B, w.L, w.H, w.dk, w.dv
    q, k, v, dO = dev(x["q"], w.dtype), dev(x["k"], w.dtype), dev(x["v"], w.dtype), dev(x["dO"], w.dtype)
    z = dev(x["z"])
    ws_f = dig.new_workspace(B, H, L, dk, dv)
    ws_b = dig.new_workspace(B, H, L, dk, dv, backward=True)
    xc = torch.randn(B, w.grid_h, w.grid_w, 64, device="cuda")
    wc = torch.randn(64, 3, 3, device="cuda")
    yc = torch.empty(B, L, 64, device="cuda")
    res = {}
    for mode in (0, 3):  # different scan orders: different gate factors, states and outputs
        o = torch.full((B, L, H, dv), float("nan"), device="cuda")
        g = tuple(torch.full(s, float("nan"), device="cuda") for s in ((B, L, H, dk), (B, L, H, dk), (B, L, H, dv)))
        dla = torch.full(tuple(z.shape), float("nan"), device="cuda")
        dig.dig_gla_fwd(q, k, v, z, w.inv_tau, o, w.grid_h, w.grid_w, mode, ws_f)
        dig.dig_srem_reorient_dwconv(xc, wc, None, yc, mode)
        dig.dig_gla_bwd_saved(q, k, v, z, w.inv_tau, dO, g[0], g[1], g[2], dla, w.grid_h, w.grid_w, mode, ws_f, ws_b)
        res[mode] = (o, g + (dla,))
    torch.cuda.synchronize()
    assert dig.dig_read_status(ws_f) == dig.DIG_OK and dig.dig_read_status(ws_b) == dig.DIG_OK
    for mode, (o, grads) in res.items():
        assert rel_err(host(o), oracle_fwd(index, mode)) <= tol(w.dtype), mode
        errs = [rel_err(host(a), r) for a, r in zip(grads, oracle_bwd(index, mode))]
        assert max(errs) <= tol(w.dtype), (mode, errs)

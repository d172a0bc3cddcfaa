"""GPU: the training step that bench.py times, checked exactly as it runs.

bench.py's step is dig_gla_fwd with bf16 o and y and the fused Swish*RMSNorm
epilogue, then dig_gla_bwd_saved on that forward's workspace with bf16 dq, dk
and dv, then the SREM conv with a bf16 output.  Each op is run here twice on the
same inputs: once with fp32 outputs, which must match the fp64 oracle within the
bf16-input bound (1e-2 of max|d| / rms), and once with the bench's bf16 outputs,
each of which must be exactly the round-to-nearest-even of its fp32 twin (the
kernels compute in fp32 and round only when they store).  d log(alpha) is fp32
in both; with one gate shared by the heads it is a sum of per-head atomics, so
it is compared with the oracle instead.
"""
import pytest
import torch

import oracle
from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import dev, host, oracle_bwd, oracle_fwd, rel_err, tol, workload_inputs

pytestmark = pytest.mark.gpu

BENCH_WORKLOADS = [3, 4]  # DiG-S/2 1792^2 (the bench step) and DiG-XL/2 2048^2 (the largest single-GPU shape)


def _step(dig, w, t, mode, odt):
    """One bench step's GLA ops with outputs of type `odt`; returns the outputs and both workspaces."""
    B, L, H, dk, dv = w.B, w.L, w.H, w.dk, w.dv
    nan = float("nan")
    o = torch.full((B, L, H, dv), nan, dtype=odt, device="cuda")
    y = torch.full_like(o, nan) if t["r"] is not None else None
    dq = torch.full((B, L, H, dk), nan, dtype=odt, device="cuda")
    dkk = torch.full_like(dq, nan)
    dvv = torch.full((B, L, H, dv), nan, dtype=odt, device="cuda")
    dla = torch.full(tuple(t["z"].shape), nan, dtype=torch.float32, device="cuda")
    ws_f = dig.new_workspace(B, H, L, dk, dv)
    ws_b = dig.new_workspace(B, H, L, dk, dv, backward=True)
    dig.dig_gla_fwd(t["q"], t["k"], t["v"], t["z"], w.inv_tau, o, w.grid_h, w.grid_w, mode, ws_f, r=t["r"], y=y)
    dig.dig_gla_bwd_saved(t["q"], t["k"], t["v"], t["z"], w.inv_tau, t["dO"], dq, dkk, dvv, dla, w.grid_h, w.grid_w,
                          mode, ws_f, ws_b)
    return (o, y, dq, dkk, dvv, dla), (ws_f, ws_b)


@pytest.mark.parametrize("index", BENCH_WORKLOADS)
@pytest.mark.parametrize("mode", range(4))
def test_bench_step_outputs(index, mode):
    from gated_linear_attention_fwd_b200 import dig
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    t = {n: dev(x[n], "bf16") for n in ("q", "k", "v", "dO")}
    t["z"] = dev(x["z"])
    t["r"] = dev(x["r"], "bf16") if w.epilogue else None  # the epilogue is part of workload 3's step only
    f32, f32_ws = _step(dig, w, t, mode, torch.float32)
    b16, b16_ws = _step(dig, w, t, mode, torch.bfloat16)
    torch.cuda.synchronize()
    for ws in f32_ws + b16_ws:
        assert dig.dig_read_status(ws) == dig.DIG_OK
    o_ref = oracle_fwd(index, mode)
    refs = (o_ref, oracle.epilogue(o_ref, x["r"]) if w.epilogue else None) + tuple(oracle_bwd(index, mode))
    names = ("o", "y", "dq", "dk", "dv", "dlogalpha")
    errs = {n: rel_err(host(g), r) for n, g, r in zip(names, f32, refs) if g is not None}
    assert max(errs.values()) <= tol(w.dtype), errs
    for n, a, b in zip(names[:5], b16[:5], f32[:5]):
        assert (a is None) == (b is None) and (a is None or torch.equal(a, b.to(torch.bfloat16))), n
    assert rel_err(host(b16[5]), refs[5]) <= tol(w.dtype)


@pytest.mark.parametrize("mode", range(4))
def test_bench_conv_output(mode):
    """The step's conv (workload 3, C = 384): bf16 in, bf16 out, as the bench runs it."""
    from gated_linear_attention_fwd_b200 import dig
    w = inputs.WORKLOADS[3]
    x = workload_inputs(3)
    xc, wc = dev(x["x_conv"], "bf16"), dev(x["w_conv"])
    y32 = torch.full((w.B, w.L, w.conv_C), float("nan"), device="cuda")
    y16 = torch.full_like(y32, float("nan"), dtype=torch.bfloat16)
    dig.dig_srem_reorient_dwconv(xc, wc, None, y32, mode)
    dig.dig_srem_reorient_dwconv(xc, wc, None, y16, mode)
    torch.cuda.synchronize()
    assert rel_err(host(y32), oracle.srem_dwconv(x["x_conv"], x["w_conv"], None, mode)) <= 1e-5
    assert torch.equal(y16, y32.to(torch.bfloat16))

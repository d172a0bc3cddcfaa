"""dig_gla_fwd_noalloc: the forward entry point that allocates nothing.

It serves callers that cannot call cudaMalloc -- plug-ins hosted by a runtime
that owns all device memory and forbids its extensions to allocate, and host
programs that link only this library with no device allocator of their own.
Instead of a caller-allocated workspace it uses a scratch array built into the
library.  This file is collected last, so a failure here leaves every other test
already run; it also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import dev, host, rel_err, tol

pytestmark = pytest.mark.gpu


def test_noalloc_forward_matches_the_workspace_forward_on_two_calls_in_a_row():
    from gated_linear_attention_fwd_b200 import dig
    # 4 x 6 sequences of 32 chunks: the gate factors and the chunk states live in
    # the built-in scratch
    w = inputs.WORKLOADS[2]
    x = inputs.make_inputs(w)
    q, k, v, z = dev(x["q"], w.dtype), dev(x["k"], w.dtype), dev(x["v"], w.dtype), dev(x["z"])
    B, L, H = w.B, w.L, w.H
    o_ref = torch.full((B, L, H, w.dv), float("nan"), device="cuda")
    ws = dig.new_workspace(B, H, L, w.dk, w.dv)
    dig.dig_gla_fwd(q, k, v, z, w.inv_tau, o_ref, w.grid_h, w.grid_w, 3, ws)
    assert dig.dig_read_status(ws) == dig.DIG_OK
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
        st = dig.lib.dig_gla_fwd_noalloc(
            ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
            ctypes.c_void_p(z.data_ptr()), 1, w.inv_tau, ctypes.c_void_p(o.data_ptr()), None, None, 1e-5, None,
            B, H, L, w.dk, w.dv, w.grid_h, w.grid_w, 3, dig.DIG_BF16, dig.DIG_F32,
            ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == dig.DIG_OK, dig.lib.dig_last_error()
        torch.cuda.synchronize()
        assert status.item() == dig.DIG_OK, "call %d: device status %d" % (call, status.item())
        assert rel_err(host(o), host(o_ref)) <= tol(w.dtype), "call %d" % call


def test_noalloc_rejects_a_shape_beyond_the_scratch():
    from gated_linear_attention_fwd_b200 import dig
    B, H, Hg, Wg, dk, dv = 64, 64, 64, 64, 64, 64      # 4096 sequences: far more than the 16 MiB scratch holds
    assert dig.gla_workspace_bytes(B, H, Hg * Wg, dk, dv) > (16 << 20)
    buf = torch.zeros(64, dtype=torch.float32, device="cuda")   # never touched: rejected before any launch
    p = ctypes.c_void_p(buf.data_ptr())
    st = dig.lib.dig_gla_fwd_noalloc(p, p, p, p, 1, 0.0625, p, None, None, 1e-5, None, B, H, Hg * Wg, dk, dv, Hg, Wg,
                                     0, dig.DIG_BF16, dig.DIG_BF16, None, None)
    assert st == dig.DIG_ERR_WORKSPACE_TOO_SMALL
    assert b"built-in scratch" in dig.lib.dig_last_error()

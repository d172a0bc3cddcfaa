"""C-ABI library checks that need no GPU: it loads, exports every function
include/dig.h declares, and rejects bad arguments on the host with the exact
status code before anything is launched."""
import ctypes
import subprocess

import pytest

from gated_linear_attention_fwd_b200 import dig

N = None


def _fwd(**kw):
    args = dict(q=1024, k=1024, v=1024, z=1024, gate_heads=1, inv_tau=1 / 16, o=1024, r=N, gamma=N, eps=1e-5,
                y=N, B=1, H=2, L=12, d_k=32, d_v=64, grid_h=3, grid_w=4, scan_mode=0, dtype=1, out_dtype=0,
                ws=4096, ws_bytes=1 << 20, stream=N)
    args.update(kw)
    a = args
    return dig.lib.dig_gla_fwd(a["q"], a["k"], a["v"], a["z"], a["gate_heads"], a["inv_tau"], a["o"], a["r"],
                               a["gamma"], a["eps"], a["y"], a["B"], a["H"], a["L"], a["d_k"], a["d_v"],
                               a["grid_h"], a["grid_w"], a["scan_mode"], a["dtype"], a["out_dtype"], a["ws"],
                               a["ws_bytes"], a["stream"])


def test_exports_every_declared_function():
    names = dig.header_functions()
    assert {"dig_gla_fwd", "dig_gla_bwd", "dig_srem_reorient_dwconv", "dig_gla_workspace_bytes",
            "dig_epilogue_bwd", "dig_srem_reorient_dwconv_bwd", "dig_gate_proj_fwd", "dig_gate_proj_bwd",
            "dig_read_status", "dig_status_string", "dig_last_error", "dig_gla_supported"} <= set(names)
    for n in names:
        assert hasattr(dig.lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", dig.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert set(names) <= exported



def test_supported_dims():
    assert dig.lib.dig_gla_supported(32, 64) == 1
    assert dig.lib.dig_gla_supported(36, 72) == 1
    assert dig.lib.dig_gla_supported(64, 64) == 1
    assert dig.lib.dig_gla_supported(48, 48) == 0


@pytest.mark.parametrize("kw, code", [
    (dict(L=13), dig.DIG_ERR_INVALID_ARGUMENT),                 # L != grid_h * grid_w
    (dict(scan_mode=4), dig.DIG_ERR_INVALID_ARGUMENT),
    (dict(scan_mode=-1), dig.DIG_ERR_INVALID_ARGUMENT),
    (dict(dtype=2), dig.DIG_ERR_INVALID_ARGUMENT),
    (dict(out_dtype=7), dig.DIG_ERR_INVALID_ARGUMENT),
    (dict(gate_heads=3), dig.DIG_ERR_INVALID_ARGUMENT),         # neither 1 nor H
    (dict(H=0), dig.DIG_ERR_INVALID_ARGUMENT),
    (dict(B=-1), dig.DIG_ERR_INVALID_ARGUMENT),
    (dict(d_k=48, d_v=48), dig.DIG_ERR_UNSUPPORTED),
    (dict(ws=N), dig.DIG_ERR_INVALID_ARGUMENT),
    (dict(ws=4100), dig.DIG_ERR_MISALIGNED),
    (dict(q=1032), dig.DIG_ERR_MISALIGNED),
    (dict(o=N), dig.DIG_ERR_INVALID_ARGUMENT),
    (dict(ws_bytes=16), dig.DIG_ERR_WORKSPACE_TOO_SMALL),
])
def test_fwd_rejects_bad_arguments_on_host(kw, code):
    assert _fwd(**kw) == code
    assert dig.lib.dig_last_error().decode()


def test_empty_problem_is_a_no_op():
    assert _fwd(B=0) == dig.DIG_OK
    assert _fwd(L=0, grid_h=0, grid_w=5) == dig.DIG_OK


def test_bwd_and_conv_reject_bad_arguments_on_host():
    st = dig.lib.dig_gla_bwd(1024, 1024, 1024, 1024, 1, 0.1, 1024, 1024, 1024, 1024, 1024,
                             1, 1, 12, 32, 64, 3, 5, 0, 1, 1, 4096, 1 << 20, N)
    assert st == dig.DIG_ERR_INVALID_ARGUMENT
    st = dig.lib.dig_gla_bwd(1024, 1024, 1024, 1024, 1, 0.1, N, 1024, 1024, 1024, 1024,
                             1, 1, 12, 32, 64, 3, 4, 0, 1, 1, 4096, 1 << 20, N)
    assert st == dig.DIG_ERR_INVALID_ARGUMENT
    # the saved-record backward: no forward workspace, a bad grid, a forward workspace too small
    st = dig.lib.dig_gla_bwd_saved(1024, 1024, 1024, 1024, 1, 0.1, 1024, 1024, 1024, 1024, 1024,
                                   1, 1, 12, 32, 64, 3, 4, 0, 1, 1, N, 0, 4096, 1 << 20, N)
    assert st == dig.DIG_ERR_INVALID_ARGUMENT
    st = dig.lib.dig_gla_bwd_saved(1024, 1024, 1024, 1024, 1, 0.1, 1024, 1024, 1024, 1024, 1024,
                                   1, 1, 12, 32, 64, 3, 5, 0, 1, 1, 8192, 1 << 20, 4096, 1 << 20, N)
    assert st == dig.DIG_ERR_INVALID_ARGUMENT
    st = dig.lib.dig_gla_bwd_saved(1024, 1024, 1024, 1024, 1, 0.1, 1024, 1024, 1024, 1024, 1024,
                                   1, 1, 12, 32, 64, 3, 4, 0, 1, 1, 8192, 16, 4096, 1 << 20, N)
    assert st == dig.DIG_ERR_WORKSPACE_TOO_SMALL
    assert dig.lib.dig_srem_reorient_dwconv(1024, 1024, N, 1024, 1, 3, 4, 8, 5, 1, 1, N) == \
        dig.DIG_ERR_INVALID_ARGUMENT
    assert dig.lib.dig_srem_reorient_dwconv(1024, 1024, N, 1032, 1, 3, 4, 8, 0, 1, 1, N) == dig.DIG_ERR_MISALIGNED
    assert dig.lib.dig_srem_reorient_dwconv(1024, 1024, N, 1024, 1, 3, 4, 0, 0, 1, 1, N) == \
        dig.DIG_ERR_INVALID_ARGUMENT


def test_backward_helpers_reject_bad_arguments_on_host():
    E = dig.lib.dig_epilogue_bwd
    ok = dict(o=1024, r=1024, gamma=N, eps=1e-5, dY=1024, d_o=1024, d_r=1024, d_gamma=N, rows=4, d_v=64,
              dtype=1, out_dtype=1)

    def epi(**kw):
        a = dict(ok, **kw)
        return E(a["o"], a["r"], a["gamma"], a["eps"], a["dY"], a["d_o"], a["d_r"], a["d_gamma"], a["rows"],
                 a["d_v"], a["dtype"], a["out_dtype"], N)
    assert epi(d_v=0) == dig.DIG_ERR_INVALID_ARGUMENT
    assert epi(rows=-1) == dig.DIG_ERR_INVALID_ARGUMENT
    assert epi(d_v=8193) == dig.DIG_ERR_UNSUPPORTED
    assert epi(eps=-1.0) == dig.DIG_ERR_INVALID_ARGUMENT
    assert epi(dtype=7) == dig.DIG_ERR_INVALID_ARGUMENT
    assert epi(o=N) == dig.DIG_ERR_INVALID_ARGUMENT
    assert epi(d_r=1032) == dig.DIG_ERR_MISALIGNED
    assert epi(d_gamma=1028) == dig.DIG_ERR_MISALIGNED
    C = dig.lib.dig_srem_reorient_dwconv_bwd
    # x, w, dY, dx, dw, dbias, B, grid_h, grid_w, C, mode, dtype, out_dtype, stream
    assert C(1024, 1024, 1024, 1024, N, N, 1, 3, 4, 0, 0, 1, 1, N) == dig.DIG_ERR_INVALID_ARGUMENT
    assert C(1024, 1024, 1024, 1024, N, N, 1, 3, 4, 8, 4, 1, 1, N) == dig.DIG_ERR_INVALID_ARGUMENT
    assert C(N, 1024, 1024, 1024, 1024, N, 1, 3, 4, 8, 0, 1, 1, N) == dig.DIG_ERR_INVALID_ARGUMENT  # dw needs x
    assert C(1024, N, 1024, 1024, N, N, 1, 3, 4, 8, 0, 1, 1, N) == dig.DIG_ERR_INVALID_ARGUMENT
    assert C(1024, 1024, 1024, 1024, 1036, N, 1, 3, 4, 8, 0, 1, 1, N) == dig.DIG_ERR_MISALIGNED
    assert C(1024, 1024, 1024, 1024, N, N, 1, 3, 4, 8, 0, 1, 2, N) == dig.DIG_ERR_INVALID_ARGUMENT


def test_gate_projection_rejects_bad_arguments_on_host():
    F, Bw = dig.lib.dig_gate_proj_fwd, dig.lib.dig_gate_proj_bwd
    # x, W1, W2, b, z, u, rows, D, R, d_k, dtype, stream
    assert F(1024, 1024, 1024, N, 1024, N, 4, 0, 16, 32, 1, N) == dig.DIG_ERR_INVALID_ARGUMENT
    assert F(1024, 1024, 1024, N, 1024, N, 4, 12, 16, 32, 1, N) == dig.DIG_ERR_UNSUPPORTED      # D % 8
    assert F(1024, 1024, 1024, N, 1024, N, 4, 384, 33, 32, 1, N) == dig.DIG_ERR_UNSUPPORTED     # R > 32
    assert F(1024, 1024, 1024, N, 1024, N, 4, 384, 16, 129, 1, N) == dig.DIG_ERR_UNSUPPORTED    # d_k > 128
    assert F(1024, 1024, 1024, N, 1024, N, 4, 8192, 32, 32, 1, N) == dig.DIG_ERR_UNSUPPORTED    # shared memory
    assert F(1024, 1024, 1024, N, N, N, 4, 384, 16, 32, 1, N) == dig.DIG_ERR_INVALID_ARGUMENT
    assert F(1024, 1024, 1024, N, 1032, N, 4, 384, 16, 32, 1, N) == dig.DIG_ERR_MISALIGNED
    assert F(1024, 1024, 1024, N, 1024, N, 4, 384, 16, 32, 9, N) == dig.DIG_ERR_INVALID_ARGUMENT
    # x, W1, W2, u, z, dla, inv_tau, dx, dW1, dW2, db, rows, D, R, d_k, dtype, out_dtype, stream
    a = [1024] * 6 + [0.0625] + [1024] * 3 + [N, 4, 384, 16, 32, 1, 1, N]    # valid (not launched here)
    bad = list(a); bad[6] = 0.0
    assert Bw(*bad) == dig.DIG_ERR_INVALID_ARGUMENT                                          # inv_tau
    bad = list(a); bad[8] = N
    assert Bw(*bad) == dig.DIG_ERR_INVALID_ARGUMENT                                          # dW1
    bad = list(a); bad[7] = 1040 + 4
    assert Bw(*bad) == dig.DIG_ERR_MISALIGNED
    bad = list(a); bad[12] = 20
    assert Bw(*bad) == dig.DIG_ERR_UNSUPPORTED                                               # D % 8


def test_workspace_bytes():
    assert dig.gla_workspace_bytes(4, 6, 4096, 32, 64) > 256
    assert dig.gla_workspace_bytes(4, 6, 4096, 32, 64, backward=True) > dig.gla_workspace_bytes(4, 6, 4096, 32, 64)
    assert dig.lib.dig_gla_workspace_bytes(1, 0, 1, 16, 32, 64, 0) == 0
    assert dig.lib.dig_gla_workspace_bytes(1, 1, 1, 16, 32, 64, 2) == 0
    assert dig.lib.dig_gla_workspace_bytes(1, 4, 3, 16, 32, 64, 0) == 0      # gate_heads neither 1 nor H
    assert dig.gla_workspace_bytes(2, 4, 256, 32, 64, gate_heads=4) > dig.gla_workspace_bytes(2, 4, 256, 32, 64)


def test_status_strings():
    for s in range(8):
        assert dig.lib.dig_status_string(s)

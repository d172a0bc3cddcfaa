"""GPU parity of the epilogue backward (dig_epilogue_bwd) and the SREM conv
backward (dig_srem_reorient_dwconv_bwd) against the fp64 oracle.

Inputs are the seeded workloads' tensors (o and dY are drawn like dO: N(0,1)
stored in the workload's dtype).  Bars: with fp32 outputs max|d|/rms(ref) <= 1e-4
(fp32 arithmetic on the exact stored inputs; the parameter gradients are fp32
sums over up to ~2.6e5 rows).  bf16 outputs are checked to be the exact
round-to-nearest-even of the same kernel's fp32 result: d_o has max/rms near 10
at the workload sizes, so one bf16 rounding alone moves it by up to ~2% of rms."""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import TORCH, dev, host, rel_err, workload_inputs

pytestmark = pytest.mark.gpu


def _store(a, dtype):
    return inputs.round_bf16(a) if dtype == "bf16" else np.asarray(a, dtype=np.float32)


def _epi_case(rows, dv, dtype, seed, with_gamma=True):
    rng = np.random.default_rng(seed)
    o = _store(rng.standard_normal((rows, dv)), dtype)
    r = _store(rng.standard_normal((rows, dv)), dtype)
    dy = _store(rng.standard_normal((rows, dv)), dtype)
    gamma = (1.0 + 0.1 * rng.standard_normal(dv)).astype(np.float32) if with_gamma else None
    return o, r, dy, gamma


def _epi_gpu(o, r, dy, gamma, dtype, out_dtype, eps=1e-5, want_gamma=True):
    from gated_linear_attention_fwd_b200 import dig
    ot, rt, dyt = dev(o, dtype), dev(r, dtype), dev(dy, dtype)
    d_o = torch.full(o.shape, float("nan"), dtype=TORCH[out_dtype], device="cuda")
    d_r = torch.full(o.shape, float("nan"), dtype=TORCH[out_dtype], device="cuda")
    d_g = torch.full((o.shape[-1],), float("nan"), dtype=torch.float32, device="cuda") if want_gamma else None
    dig.dig_epilogue_bwd(ot, rt, dyt, d_o, d_r, None if gamma is None else dev(gamma), eps, d_g)
    torch.cuda.synchronize()
    return d_o, d_r, d_g


def _check_epi(o, r, dy, gamma, dtype, eps=1e-5):
    ref_o, ref_r, ref_g = oracle.epilogue_bwd(o, r, dy, gamma, eps=eps)
    d_o, d_r, d_g = _epi_gpu(o, r, dy, gamma, dtype, "f32", eps)
    assert rel_err(host(d_o), ref_o) <= 1e-4
    assert rel_err(host(d_r), ref_r) <= 1e-4
    assert rel_err(host(d_g), ref_g) <= 1e-4
    b_o, b_r, b_g = _epi_gpu(o, r, dy, gamma, dtype, "bf16", eps)
    assert torch.equal(b_o, d_o.to(torch.bfloat16)) and torch.equal(b_r, d_r.to(torch.bfloat16))
    assert rel_err(host(b_g), ref_g) <= 1e-4


@pytest.mark.parametrize("index", [3, 4, 0])
def test_epilogue_bwd_workloads(index):
    """DiG-S/2 1792^2 (d_v 64), DiG-XL/2 2048^2 (d_v 72) and the fp32 tiny case at full size."""
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    rows = w.B * w.L * w.H
    o, _, dy, gamma = _epi_case(rows, w.dv, w.dtype, 90 + index)
    r = x["r"] if "r" in x else _epi_case(rows, w.dv, w.dtype, 95 + index)[1]
    _check_epi(o, r.reshape(rows, w.dv), dy, gamma, w.dtype)


@pytest.mark.parametrize("rows,dv", [(1, 4), (7, 12), (6, 24), (2, 16), (33, 64), (5, 72), (300, 128), (9, 10), (4, 200), (3, 6)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_epilogue_bwd_shapes(rows, dv, dtype):
    """Every row-group width (d_v/4 up to 4, 8, 16, 32), the any-d_v path (d_v not a
    multiple of 4, or above 128) and ragged row counts."""
    o, r, dy, gamma = _epi_case(rows, dv, dtype, rows * 1000 + dv)
    _check_epi(o, r, dy, gamma, dtype)


def test_epilogue_bwd_without_gamma_and_large_eps():
    o, r, dy, _ = _epi_case(1000, 64, "bf16", 7, with_gamma=False)
    o[3] = 0.0                                        # an all-zero row: the norm is eps-limited
    _check_epi(o, r, dy, None, "bf16", eps=0.5)


def test_epilogue_bwd_saturated_gates():
    """r far in both tails: sigmoid -> 0 and 1 without overflow."""
    o, r, dy, gamma = _epi_case(64, 64, "f32", 8)
    r = np.where(np.arange(64)[None, :] % 2 == 0, 60.0, -60.0).astype(np.float32) * np.ones_like(r)
    _check_epi(o, r, dy, gamma, "f32")


def test_epilogue_bwd_zero_rows_clears_d_gamma():
    from gated_linear_attention_fwd_b200 import dig
    e = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    d_g = torch.full((64,), 5.0, device="cuda")
    dig.dig_epilogue_bwd(e, e, e, e.clone(), e.clone(), None, 1e-5, d_g)
    torch.cuda.synchronize()
    assert torch.all(d_g == 0)


# ----------------------------------------------------------------------------- conv backward

def _conv_bwd_gpu(x, w, dy, mode, dtype, out_dtype, want_w=True):
    from gated_linear_attention_fwd_b200 import dig
    B, Hg, Wg, C = x.shape
    dx = torch.full((B, Hg, Wg, C), float("nan"), dtype=TORCH[out_dtype], device="cuda")
    dw = torch.full((C, 3, 3), float("nan"), device="cuda") if want_w else None
    db = torch.full((C,), float("nan"), device="cuda") if want_w else None
    dig.dig_srem_reorient_dwconv_bwd(dev(x, dtype) if want_w else None, dev(w), dev(dy, dtype), dx, mode, dw, db)
    torch.cuda.synchronize()
    return dx, dw, db


def _check_conv_bwd(x, w, dy, mode, dtype):
    ref_dx, ref_dw, ref_db = oracle.srem_dwconv_bwd(x, w, dy, mode)
    dx, dw, db = _conv_bwd_gpu(x, w, dy, mode, dtype, "f32")
    assert rel_err(host(dx), ref_dx) <= 1e-5
    assert rel_err(host(dw), ref_dw) <= 1e-4
    assert rel_err(host(db), ref_db) <= 1e-4
    dx16, _, _ = _conv_bwd_gpu(x, w, dy, mode, dtype, "bf16", want_w=False)
    assert torch.equal(dx16, dx.to(torch.bfloat16))


@pytest.mark.parametrize("index", [0, 3])
@pytest.mark.parametrize("mode", range(4))
def test_conv_bwd_matches_oracle(index, mode):
    """The tiny fp32 case (C 64, 16x16) and DiG-S/2 1792^2 (C 384, 112x112, bf16) at full size."""
    wl = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    rng = np.random.default_rng(100 + mode)
    dy = _store(rng.standard_normal((wl.B, wl.L, x["x_conv"].shape[-1])), wl.dtype)
    _check_conv_bwd(x["x_conv"], x["w_conv"], dy, mode, wl.dtype)


@pytest.mark.parametrize("shape", [(1, 1, 1, 8), (2, 5, 3, 24), (1, 7, 9, 5), (3, 1, 17, 16), (1, 9, 11, 66),
                                   (2, 4, 4, 2), (1, 13, 6, 130)])
@pytest.mark.parametrize("mode", [0, 1, 2, 3])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_conv_bwd_edge_shapes(shape, mode, dtype):
    """Single pixels, single rows and columns, ragged tiles, odd C (per-element path),
    channel slabs that are partly filled (C 66, 130) and C = 2."""
    rng = np.random.default_rng(sum(shape) + 7 * mode)
    B, Hg, Wg, C = shape
    x = _store(rng.standard_normal(shape), dtype)
    w = rng.standard_normal((C, 3, 3)).astype(np.float32)
    dy = _store(rng.standard_normal((B, Hg * Wg, C)), dtype)
    _check_conv_bwd(x, w, dy, mode, dtype)


def test_conv_bwd_identity_kernel_is_exact_inverse_reorient():
    """With the identity kernel dx is dY put back in grid order: bit-exact."""
    rng = np.random.default_rng(3)
    B, Hg, Wg, C = 2, 112, 112, 384
    w = np.zeros((C, 3, 3), dtype=np.float32)
    w[:, 1, 1] = 1.0
    dy = inputs.round_bf16(rng.standard_normal((B, Hg * Wg, C)))
    for mode in range(4):
        dx, _, _ = _conv_bwd_gpu(np.zeros((B, Hg, Wg, C), np.float32), w, dy, mode, "bf16", "bf16", want_w=False)
        perm = oracle.scan_index(mode, Hg, Wg)
        ref = np.zeros((B, Hg * Wg, C), dtype=np.float32)
        ref[:, perm] = dy
        assert torch.equal(dx.float().cpu(), torch.from_numpy(ref.reshape(B, Hg, Wg, C)))


def test_conv_bwd_empty_grid_clears_parameter_gradients():
    from gated_linear_attention_fwd_b200 import dig
    C = 6
    x = torch.empty((0, 4, 4, C), dtype=torch.bfloat16, device="cuda")
    dw = torch.full((C, 3, 3), 3.0, device="cuda")
    db = torch.full((C,), 3.0, device="cuda")
    dig.dig_srem_reorient_dwconv_bwd(x, dev(np.ones((C, 3, 3))), torch.empty((0, 16, C), dtype=torch.bfloat16,
                                                                             device="cuda"),
                                     x.clone(), 0, dw, db)
    torch.cuda.synchronize()
    assert torch.all(dw == 0) and torch.all(db == 0)

"""GPU parity of dig_srem_reorient_dwconv against the oracle.

The identity-initialised kernel makes SREM a pure reorient permutation, which
must be bit-exact; general weights must agree to fp32 rounding."""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_attention_fwd_b200 import inputs
from tests.gpu_helpers import dev, host, rel_err, workload_inputs

pytestmark = pytest.mark.gpu


def _conv(x, w, bias, mode, in_dtype, out_dtype):
    from gated_linear_attention_fwd_b200 import dig
    B, Hg, Wg, C = x.shape
    xt = dev(x, in_dtype)
    y = torch.full((B, Hg * Wg, C), float("nan"), dtype=torch.float32 if out_dtype == "f32" else torch.bfloat16,
                   device="cuda")
    dig.dig_srem_reorient_dwconv(xt, dev(w), None if bias is None else dev(bias), y, mode)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("index", [0, 3])
@pytest.mark.parametrize("mode", range(4))
def test_conv_matches_oracle(index, mode):
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    y = _conv(x["x_conv"], x["w_conv"], None, mode, w.dtype, "f32")
    ref = oracle.srem_dwconv(x["x_conv"], x["w_conv"], None, mode)
    assert rel_err(host(y), ref) <= 1e-5
    y16 = _conv(x["x_conv"], x["w_conv"], None, mode, w.dtype, "bf16")
    assert torch.equal(y16, y.to(torch.bfloat16))


@pytest.mark.parametrize("mode", range(4))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_identity_kernel_is_exact_reorient(mode, dtype):
    rng = np.random.default_rng(mode)
    B, Hg, Wg, C = 2, 112, 112, 384
    x = inputs.round_bf16(rng.standard_normal((B, Hg, Wg, C))) if dtype == "bf16" else \
        rng.standard_normal((B, Hg, Wg, C)).astype(np.float32)
    wid = np.zeros((C, 3, 3), dtype=np.float32)
    wid[:, 1, 1] = 1.0
    y = _conv(x, wid, None, mode, dtype, dtype)
    perm = oracle.scan_index(mode, Hg, Wg)
    ref = torch.from_numpy(np.ascontiguousarray(x.reshape(B, Hg * Wg, C)[:, perm])).cuda()
    assert torch.equal(y.float(), ref.float())


@pytest.mark.parametrize("shape", [(1, 1, 1, 8), (2, 5, 3, 24), (1, 7, 9, 5), (3, 1, 17, 16)])
@pytest.mark.parametrize("mode", [0, 2, 3])
def test_conv_edge_shapes_with_bias(shape, mode):
    rng = np.random.default_rng(sum(shape))
    B, Hg, Wg, C = shape
    x = inputs.round_bf16(rng.standard_normal(shape))
    wts = rng.standard_normal((C, 3, 3)).astype(np.float32)
    bias = rng.standard_normal(C).astype(np.float32)
    y = _conv(x, wts, bias, mode, "bf16", "f32")
    ref = oracle.srem_dwconv(x, wts, bias, mode)
    assert rel_err(host(y), ref) <= 1e-5

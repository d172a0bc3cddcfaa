"""The synthetic DiG block (gated_linear_attention_fwd_b200.dig_block), step by
step, against float64 references of its steps: the oracle's gate projection,
GLA recurrence, output-gate epilogue and SREM convolution, and numpy for the
block's dense projections, norms, activations and residuals.  Each step is
checked on the block's own inputs to that step (the buffers it leaves), so
rounding does not accumulate across steps; every buffer the block stores in bf16
must be within two bf16 units in the last place of the reference, plus a small
absolute slack (1e-3 of the reference's rms; 1e-2 for the GLA output, the bf16
parity bound of the recurrence itself; 2e-2 after the GELU, whose slope carries a
1-ulp difference of its bf16 input into its small outputs).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import host

pytestmark = pytest.mark.gpu


def bf16(a):
    """Round-to-nearest-even to bf16, returned as float64."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def rmsnorm(x, eps=1e-6):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def gelu(a):
    return 0.5 * a * (1.0 + np.tanh(0.7978845608028654 * (a + 0.044715 * a ** 3)))


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def close(name, got, ref, slack=1e-3):
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64).reshape(np.shape(got))
    rms = np.sqrt(np.mean(ref * ref))
    bound = 2.0 * 2.0 ** -8 * np.abs(ref) + slack * rms
    bad = np.abs(got - ref) > bound
    assert not bad.any(), "%s: %d of %d outside 2 bf16 ulp + %.0e rms (worst %.3e)" % (
        name, int(bad.sum()), bad.size, slack, float(np.max(np.abs(got - ref) - bound)))


@pytest.mark.parametrize("layer", [0, 3])
def test_dig_block_steps_match_their_references(layer):
    from gated_linear_attention_fwd_b200 import dig_block
    B, Hg, Wg = 2, 16, 24
    L = Hg * Wg
    blk = dig_block.dig_s2(Hg, Wg, layer=layer, seed=3)
    D, H, dk, dv = blk.D, blk.H, blk.d_k, blk.d_v
    g = torch.Generator(device="cpu").manual_seed(17)
    x0 = torch.randn(B, L, D, generator=g).to("cuda", torch.bfloat16)
    cond = torch.randn(B, D, generator=g).to("cuda", torch.bfloat16)
    buf = blk.buffers(B, L, "cuda")
    x = x0.clone()
    out = blk.forward(x, cond, buf)
    torch.cuda.synchronize()
    gb = {n: host(t) for n, t in buf.items() if n != "ws"}

    xr = f64(x0)
    close("SiLU(cond)", gb["c"], bf16(f64(cond) / (1.0 + np.exp(-f64(cond)))))
    mod = gb["c"] @ f64(blk.W_ada) + f64(blk.b_ada)
    assert np.max(np.abs(gb["mod"] - mod)) <= 1e-4 * np.sqrt(np.mean(mod * mod))
    sh1, sc1, g1, sh2, sc2, g2 = (gb["mod"][:, None, i * D:(i + 1) * D] for i in range(6))
    h1 = bf16(rmsnorm(xr) * (1 + sc1) + sh1)
    for n, W in (("q", blk.W_q), ("k", blk.W_k), ("v", blk.W_v), ("r", blk.W_r)):
        close(n, gb[n].reshape(B, L, -1), bf16(h1 @ f64(W)), slack=4e-3)
    z, _ = oracle.gate_proj_fwd(bf16(h1), f64(blk.W_a1), f64(blk.W_a2), f64(blk.b_a))
    assert np.max(np.abs(gb["z"].reshape(B, L, dk) - z)) <= 1e-2 * np.sqrt(np.mean(z * z))
    o = oracle.gla_fwd(gb["q"], gb["k"], gb["v"], gb["z"], blk.inv_tau, Hg, Wg, blk.scan_mode)
    close("o", gb["o"], o, slack=1e-2)
    close("y", gb["y"], oracle.epilogue(o, gb["r"], f64(blk.gamma), eps=1e-5), slack=1e-2)
    close("attn", gb["attn"], bf16(gb["y"].reshape(B, L, H * dv) @ f64(blk.W_o)))
    x1 = bf16(xr + g1 * gb["attn"])
    close("h2", gb["h"], bf16(rmsnorm(x1) * (1 + sc2) + sh2))
    # the GELU acts on the bf16-rounded product, whose 1-ulp flips its slope carries over
    close("f1", gb["f1"], bf16(gelu(bf16(gb["h"] @ f64(blk.W_1)))), slack=2e-2)
    close("f2", gb["f2"], bf16(gb["f1"] @ f64(blk.W_2)))
    close("x2", host(x), bf16(x1 + g2 * gb["f2"]))
    close("out", host(out), bf16(oracle.srem_dwconv(host(x).reshape(B, Hg, Wg, D), f64(blk.w_conv), None, 0)))

"""A synthetic DiG block forward around the library's token mixer.

The block follows the DiG slides' Fig. 4 and the "DiG Block" section of the
paper: the conditioning (timestep + label embedding) regresses, through SiLU and
a linear layer, the adaLN shift / scale / gate pairs of the two branches; the
token-mixer branch is RMSNorm, modulation, the GLA layer (q, k, v, the output
gate r and the low-rank key gate from the normalised tokens; the GLA recurrence
in the layer's scan order with the Swish(r) * RMSNorm(o) output gate; the output
projection) and a gated residual; the feed-forward branch is RMSNorm,
modulation, a GELU MLP and a gated residual; the SREM then runs its 3 x 3
depthwise convolution over the token grid.

Readings where the pages leave the step open (each the plainest one):
  * tokens stay in grid order between blocks: a layer's scan direction is the
    GLA call's scan mode (the permutation is fused into the kernels' loads), so
    the SREM convolution writes grid order (its scan mode 0);
  * the SREM convolution is applied to the block output directly (identity
    initialised: centre tap 1, the rest 0, so a fresh block passes its tokens
    through), without a residual of its own;
  * the adaLN modulation is x * (1 + scale) + shift after an RMSNorm without a
    learnable weight; the FFN hidden size is 4 D.

Random weights (seeded); no trained weights exist here and none are needed to
time the mixer in its block.  Dense projections are library GEMMs (torch.matmul /
addmm, i.e. cuBLAS, with the fp32 copy of the tiny [B, D] conditioning that the
adaLN projection takes); every other step runs in libdig.so's kernels.
"""
from __future__ import annotations

import torch

from . import dig


class DiGBlock:
    def __init__(self, D, H, d_k, d_v, rank, grid_h, grid_w, scan_mode, seed=0, device="cuda", inv_tau=1.0 / 16.0,
                 ffn_mult=4):
        g = torch.Generator(device="cpu").manual_seed(seed)

        def w(*shape, std=0.02, dtype=torch.bfloat16):
            return (torch.randn(*shape, generator=g) * std).to(device=device, dtype=dtype).contiguous()

        self.D, self.H, self.d_k, self.d_v, self.rank = D, H, d_k, d_v, rank
        self.grid_h, self.grid_w, self.scan_mode, self.inv_tau = grid_h, grid_w, scan_mode, inv_tau
        self.W_ada = w(D, 6 * D, dtype=torch.float32)
        self.b_ada = w(6 * D, dtype=torch.float32)
        # q and k at d_k^(-1/4) each, so that q . k has unit variance over d_k channels
        qk_std = D ** -0.5 * d_k ** -0.25
        self.W_q, self.W_k = w(D, H * d_k, std=qk_std), w(D, H * d_k, std=qk_std)
        self.W_v, self.W_r = w(D, H * d_v, std=D ** -0.5), w(D, H * d_v, std=D ** -0.5)
        self.W_a1 = w(D, rank, dtype=torch.float32)
        self.W_a2 = w(rank, d_k, dtype=torch.float32)
        self.b_a = torch.zeros(d_k, device=device, dtype=torch.float32)
        self.gamma = torch.ones(d_v, device=device, dtype=torch.float32)
        self.W_o = w(H * d_v, D, std=(H * d_v) ** -0.5)
        self.W_1 = w(D, ffn_mult * D, std=D ** -0.5)
        self.W_2 = w(ffn_mult * D, D, std=(ffn_mult * D) ** -0.5)
        conv = torch.zeros(D, 3, 3)
        conv[:, 1, 1] = 1.0  # identity initialisation
        self.w_conv = (conv + 0.01 * torch.randn(D, 3, 3, generator=g)).to(device=device).contiguous()

    def buffers(self, B, L, device):
        """Activations of one call (allocated once per shape)."""
        D, H, dk, dv = self.D, self.H, self.d_k, self.d_v
        bf = torch.bfloat16
        e = lambda *s, dt=bf: torch.empty(*s, device=device, dtype=dt)
        return {"c": e(B, D), "mod": e(B, 6 * D, dt=torch.float32), "h": e(B, L, D),
                "q": e(B, L, H, dk), "k": e(B, L, H, dk), "v": e(B, L, H, dv), "r": e(B, L, H, dv),
                "z": e(B, L, 1, dk, dt=torch.float32), "u": e(B * L, self.rank, dt=torch.float32),
                "o": e(B, L, H, dv), "y": e(B, L, H, dv), "attn": e(B, L, D), "f1": e(B, L, 4 * D),
                "f2": e(B, L, D), "out": e(B, L, D),
                "ws": dig.new_workspace(B, H, L, dk, dv, device=device)}

    def forward(self, x, cond, buf, stream=None, timing=None):
        """x [B, L, D] bf16 (grid order; updated in place by the residuals), cond [B, D]
        bf16 conditioning; returns buf["out"] [B, L, D] bf16 (grid order).  With
        `timing` (a dict) the mixer's share is bracketed by CUDA events."""
        B, L, D = x.shape
        H, dk, dv = self.H, self.d_k, self.d_v
        mm = lambda a, b, out: torch.matmul(a, b, out=out)
        c = buf["c"]
        c.copy_(cond)
        dig.dig_block_activation(c, 0, stream)                              # SiLU(cond)
        torch.addmm(self.b_ada, c.float(), self.W_ada, out=buf["mod"])     # [B, 6D] adaLN parameters
        mod = buf["mod"]
        sh1, sc1, g1, sh2, sc2, g2 = (mod[:, i * D:(i + 1) * D] for i in range(6))
        h = buf["h"]
        dig.dig_block_rmsnorm_modulate(x, sh1, sc1, h, stream=stream)
        h2d = h.view(B * L, D)
        mm(h2d, self.W_q, buf["q"].view(B * L, H * dk))
        mm(h2d, self.W_k, buf["k"].view(B * L, H * dk))
        mm(h2d, self.W_v, buf["v"].view(B * L, H * dv))
        mm(h2d, self.W_r, buf["r"].view(B * L, H * dv))
        dig.dig_gate_proj_fwd(h2d, self.W_a1, self.W_a2, buf["z"].view(B * L, dk), b=self.b_a, u=buf["u"],
                              stream=stream)
        ev = None
        if timing is not None:
            ev = [torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
            ev[0].record()
        dig.dig_gla_fwd(buf["q"], buf["k"], buf["v"], buf["z"], self.inv_tau, buf["o"], self.grid_h, self.grid_w,
                        self.scan_mode, buf["ws"], r=buf["r"], gamma=self.gamma, eps=1e-5, y=buf["y"],
                        stream=stream)
        if ev is not None:
            ev[1].record()
            timing.setdefault("mixer_events", []).append(ev)
        mm(buf["y"].view(B * L, H * dv), self.W_o, buf["attn"].view(B * L, D))
        dig.dig_block_gated_add(x, g1, buf["attn"], stream)
        dig.dig_block_rmsnorm_modulate(x, sh2, sc2, h, stream=stream)
        mm(h2d, self.W_1, buf["f1"].view(B * L, 4 * D))
        dig.dig_block_activation(buf["f1"], 1, stream)                      # GELU
        mm(buf["f1"].view(B * L, 4 * D), self.W_2, buf["f2"].view(B * L, D))
        dig.dig_block_gated_add(x, g2, buf["f2"], stream)
        dig.dig_srem_reorient_dwconv(x.view(B, self.grid_h, self.grid_w, D), self.w_conv, None, buf["out"], 0,
                                     stream=stream)
        return buf["out"]


def dig_s2(grid_h, grid_w, layer=0, seed=0, device="cuda"):
    """A DiG-S/2 block (D 384, 6 heads, d_k 32, d_v 64, gate rank 16) whose scan
    order is the layer's (row-fwd, row-rev, col-fwd, col-rev for layers 0..3)."""
    return DiGBlock(384, 6, 32, 64, 16, grid_h, grid_w, layer % 4, seed=seed, device=device)


def dig_xl2(grid_h, grid_w, layer=0, seed=0, device="cuda"):
    """A DiG-XL/2 block (D 1152, 16 heads, d_k 36, d_v 72, gate rank 16)."""
    return DiGBlock(1152, 16, 36, 72, 16, grid_h, grid_w, layer % 4, seed=seed, device=device)


def model_flops(block: DiGBlock, B, L) -> float:
    """Dense-projection multiply-adds x 2 of one block call (the GEMM part)."""
    D, H, dk, dv = block.D, block.H, block.d_k, block.d_v
    per_tok = D * (2 * H * dk + 2 * H * dv) + H * dv * D + 2 * 4 * D * D + D * block.rank
    return 2.0 * B * L * per_tok + 2.0 * B * D * 6 * D


__all__ = ["DiGBlock", "dig_s2", "dig_xl2", "model_flops"]

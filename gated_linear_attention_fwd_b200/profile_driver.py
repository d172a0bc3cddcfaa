"""Run one DiG op a few times on a synthetic workload, for profilers (ncu).

    python -m gated_linear_attention_fwd_b200.profile_driver --op bwd --workload 3 --iters 4

Inputs are random tensors of the workload's shapes (values do not affect the
timing of these kernels); the device status word is checked at the end.
"""
import argparse

import torch

from . import dig, inputs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["fwd", "bwd", "conv", "epi_bwd", "conv_bwd", "gate_fwd", "gate_bwd"],
                    default="fwd")
    ap.add_argument("--workload", type=int, default=3)
    ap.add_argument("--iters", type=int, default=4)
    ap.add_argument("--mode", type=int, default=0)
    ap.add_argument("--epilogue", action="store_true")
    args = ap.parse_args()
    w = inputs.WORKLOADS[args.workload]
    B, L, H, dk, dv = w.B, w.L, w.H, w.dk, w.dv
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    g = torch.Generator(device="cuda").manual_seed(0)
    rnd = lambda *s: torch.randn(*s, device="cuda", generator=g).to(dt)
    if args.op == "conv":
        C = w.conv_C or H * dv
        x, wc = rnd(B, w.grid_h, w.grid_w, C), torch.randn(C, 3, 3, device="cuda", generator=g) * 0.1
        y = torch.empty(B, L, C, device="cuda", dtype=dt)
        for _ in range(args.iters):
            dig.dig_srem_reorient_dwconv(x, wc, None, y, args.mode)
        torch.cuda.synchronize()
        print("ok")
        return
    if args.op == "conv_bwd":
        C = w.conv_C or H * dv
        x, wc = rnd(B, w.grid_h, w.grid_w, C), torch.randn(C, 3, 3, device="cuda", generator=g) * 0.1
        dy, dx = rnd(B, L, C), torch.empty(B, w.grid_h, w.grid_w, C, device="cuda", dtype=dt)
        dw, db = torch.empty(C, 3, 3, device="cuda"), torch.empty(C, device="cuda")
        for _ in range(args.iters):
            dig.dig_srem_reorient_dwconv_bwd(x, wc, dy, dx, args.mode, dw, db)
        torch.cuda.synchronize()
        print("ok")
        return
    if args.op in ("gate_fwd", "gate_bwd"):
        D, R = w.D or 384, w.rank
        xg = rnd(B * L, D)
        W1 = 0.02 * torch.randn(D, R, device="cuda", generator=g)
        W2 = 0.02 * torch.randn(R, dk, device="cuda", generator=g)
        zg, ug = torch.empty(B * L, dk, device="cuda"), torch.empty(B * L, R, device="cuda")
        dig.dig_gate_proj_fwd(xg, W1, W2, zg, None, ug)
        dla = torch.randn(B * L, dk, device="cuda", generator=g)
        dxg, dW1, dW2 = torch.empty_like(xg), torch.empty_like(W1), torch.empty_like(W2)
        for _ in range(args.iters):
            if args.op == "gate_fwd":
                dig.dig_gate_proj_fwd(xg, W1, W2, zg, None, ug)
            else:
                dig.dig_gate_proj_bwd(xg, W1, W2, ug, zg, dla, w.inv_tau, dxg, dW1, dW2)
        torch.cuda.synchronize()
        print("ok")
        return
    if args.op == "epi_bwd":
        o, r, dy = rnd(B, L, H, dv), rnd(B, L, H, dv), rnd(B, L, H, dv)
        d_o, d_r, d_g = torch.empty_like(o), torch.empty_like(o), torch.empty(dv, device="cuda")
        for _ in range(args.iters):
            dig.dig_epilogue_bwd(o, r, dy, d_o, d_r, None, 1e-5, d_g)
        torch.cuda.synchronize()
        print("ok")
        return
    q, k, v = rnd(B, L, H, dk), rnd(B, L, H, dk), rnd(B, L, H, dv)
    z = 0.03 * torch.randn(B, L, 1, dk, device="cuda", generator=g)
    if args.op == "fwd":
        o = torch.empty(B, L, H, dv, device="cuda", dtype=dt)
        r = rnd(B, L, H, dv) if args.epilogue else None
        y = torch.empty_like(o) if args.epilogue else None
        ws = dig.new_workspace(B, H, L, dk, dv)
        for _ in range(args.iters):
            dig.dig_gla_fwd(q, k, v, z, w.inv_tau, o, w.grid_h, w.grid_w, args.mode, ws, r=r, y=y)
    else:
        # a training step's backward: the forward runs first and its records are reused
        dO = rnd(B, L, H, dv)
        dq, dkk, dvv, dla = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(z)
        o = torch.empty(B, L, H, dv, device="cuda", dtype=dt)
        fws = dig.new_workspace(B, H, L, dk, dv)
        dig.dig_gla_fwd(q, k, v, z, w.inv_tau, o, w.grid_h, w.grid_w, args.mode, fws)
        ws = dig.new_workspace(B, H, L, dk, dv, backward=True)
        for _ in range(args.iters):
            dig.dig_gla_bwd_saved(q, k, v, z, w.inv_tau, dO, dq, dkk, dvv, dla, w.grid_h, w.grid_w, args.mode, fws, ws)
    st = dig.dig_read_status(ws)
    if st != dig.DIG_OK:
        raise SystemExit("device status %d" % st)
    print("ok")


if __name__ == "__main__":
    main()

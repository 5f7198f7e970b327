"""Run one libgdr2.so kernel on its benchmark workload, for profilers.

    python -m gated_delta_rule_wy_b200.profile_cases {fwd,decode,bwd,prologue} [--launches N] [--batch B] [--epilogue]
        [--recompute]

fwd     gdr2_forward   B=4 H=16 T=4096 d=128 bf16 (the 1.3B-model layer)
decode  gdr2_decode_step  256 sequences x 16 heads, d=128, fp32 state (256 MiB)
bwd     gdr2_backward  B=2 H=16 T=4096 d=128 bf16 with saved chunk states
prologue  gdr2_block_prologue  B=4 H=16 T=4096 d=128 bf16, width-4 convolutions

Inputs are drawn once (seeded) and stay on the device; the kernel is then
launched N times back to back (use ncu -s/-c to pick one launch). --batch
overrides B of the forward and backward cases (a smaller capture whose inputs
still exceed the 126 MB L2 at B >= 2). --epilogue runs the forward with the block's
output epilogue (RMSNorm weight and SiLU gate, seeded like the bench's). --recompute runs
the backward without saved chunk states (the call recomputes them).
"""
from __future__ import annotations

import argparse

import torch

from . import inputs as I
from .binding import gdr2_backward, gdr2_decode_step, gdr2_forward, gdr2_forward_workspace_bytes, gdr2_sync_status


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=("fwd", "decode", "bwd", "prologue"))
    ap.add_argument("--launches", type=int, default=2)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--epilogue", action="store_true")
    ap.add_argument("--recompute", action="store_true")
    args = ap.parse_args()
    torch.cuda.set_device(0)
    if args.kernel == "fwd":
        c = dict(I.FWD_1P3B_BF16)
        if args.batch:
            c["B"] = args.batch
        x = I.make_forward_inputs(**c).to("cuda")
        o = torch.empty_like(x.v)
        ws = torch.empty(gdr2_forward_workspace_bytes(c["B"], c["T"], c["H"], c["dk"], c["dv"], c["dtype"]),
                         dtype=torch.uint8, device="cuda")
        g = wt = None
        if args.epilogue:
            g, wt = I.make_epilogue_inputs((c["B"], c["T"], c["H"], c["dv"]), c["dv"], seed=1009)
            g, wt = g.to("cuda"), wt.to("cuda")
        for _ in range(args.launches):
            gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, None, out=o, workspace=ws, out_gate=g,
                         norm_weight=wt)
    elif args.kernel == "decode":
        c = I.DECODE_1P3B
        gen = torch.Generator(device="cuda").manual_seed(c["seed"])
        S = torch.randn((c["N"], c["H"], c["dk"], c["dv"]), device="cuda", generator=gen) * c["state_std"]
        tok = I.make_token_inputs((c["N"], c["H"], c["dk"]), (c["N"], c["H"], c["dv"]), c["dtype"],
                                  c["decay_shift"], gen)
        for _ in range(args.launches):
            gdr2_decode_step(*tok, S)
    elif args.kernel == "prologue":
        from .binding import gdr2_block_prologue

        c = dict(I.FWD_1P3B_BF16)
        if args.batch:
            c["B"] = args.batch
        pin = {k: v.to("cuda") for k, v in I.make_prologue_inputs(c["B"], c["T"], c["H"], c["dk"], c["dv"], 4,
                                                                   c["dtype"], seed=1010).items()}
        for _ in range(args.launches):
            gdr2_block_prologue(pin["xq"], pin["xk"], pin["xv"], pin["conv_q"], pin["conv_k"], pin["conv_v"],
                                pin["a"], pin["b"], pin["w"])
    else:
        c = dict(I.BWD_1P3B_BF16)
        if args.batch:
            c["B"] = args.batch
        x = I.make_forward_inputs(**c).to("cuda")
        dO = I.make_upstream_grad(c["B"], c["T"], c["H"], c["dv"], c["seed"], dtype=c["dtype"]).cuda()
        _, _, saved = gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, None, save_states=True)
        for _ in range(args.launches):
            gdr2_backward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, dO, None, None, None if args.recompute else saved)
    gdr2_sync_status()
    print(f"profile_cases {args.kernel}: {args.launches} launches ok")


if __name__ == "__main__":
    main()

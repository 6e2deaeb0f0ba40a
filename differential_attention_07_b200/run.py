"""Run one workload a few times through the C ABI (for profilers).

    python -m differential_attention_07_b200.run --workload motif4k --iters 4
    python -m differential_attention_07_b200.run --workload decode --batch 8
    python -m differential_attention_07_b200.run --workload motif4k --batch 1 --backward

Inputs are the seeded synthetic tensors of the named workload, optionally with
a smaller batch; nothing is timed or checked, the process just launches the
kernels `--iters` times and exits 0 when the device reports no error.  With
`--backward` each iteration is the forward that saves the backward's state
followed by the backward pass (prefill workloads without grouping only).
"""
import argparse
import dataclasses
import sys

import torch

from . import inputs, ops


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="motif4k", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--batch", type=int, default=0, help="override the batch size")
    ap.add_argument("--iters", type=int, default=4)
    ap.add_argument("--backward", action="store_true", help="run the saving forward and the backward pass")
    args = ap.parse_args(argv)
    w = inputs.WORKLOADS[args.workload]
    if args.batch:
        w = dataclasses.replace(w, B=args.batch)
    x = {k: v.cuda() for k, v in inputs.workload_inputs(w).items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if args.backward:
        if w.kind != "prefill":
            print("--backward needs a prefill workload", file=sys.stderr)
            return 2
        dy = inputs.grad_output(w.B, w.N, w.H, w.dv, seed=w.seed).cuda()
        save = torch.empty(ops.fwd_save_size(w.B, w.N, w.H), dtype=torch.uint8, device="cuda")
    for _ in range(args.iters):
        if w.kind == "decode":
            ops.diffattn_decode(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                                scale=w.scale, eps=w.eps, dev_status=st)
        elif args.backward:
            ops.diffattn_fwd(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                             scale=w.scale, eps=w.eps, causal=w.causal, save=save, dev_status=st)
            ops.diffattn_bwd(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"], dy,
                             save, scale=w.scale, eps=w.eps, causal=w.causal, dev_status=st)
        else:
            f = ops.diffattn_grouped_fwd if w.kind == "grouped" else ops.diffattn_fwd
            f(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"], scale=w.scale,
              eps=w.eps, causal=w.causal, dev_status=st, window=w.window, rope_theta=w.rope_theta,
              lam_logits=x.get("lam_logits"), gate=x.get("gate"), apply_norm=w.apply_norm)
    torch.cuda.synchronize()
    if st.item() != 0:
        print(f"device status {st.item()}", file=sys.stderr)
        return 1
    print(f"ran {args.iters} x {w.name} (B={w.B}){' forward + backward' if args.backward else ''}")
    return 0


if __name__ == "__main__":
    sys.exit(main())

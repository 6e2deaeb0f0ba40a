"""Run one workload a few times through the C ABI (for profilers).

    python -m differential_attention_07_b200.run --workload motif4k --iters 4
    python -m differential_attention_07_b200.run --workload decode --batch 8

Inputs are the seeded synthetic tensors of the named workload, optionally with
a smaller batch; nothing is timed or checked, the process just launches the
kernels `--iters` times and exits 0 when the device reports no error.
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
    args = ap.parse_args(argv)
    w = inputs.WORKLOADS[args.workload]
    if args.batch:
        w = dataclasses.replace(w, B=args.batch)
    x = {k: v.cuda() for k, v in inputs.workload_inputs(w).items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(args.iters):
        if w.kind == "decode":
            ops.diffattn_decode(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                                scale=w.scale, eps=w.eps, dev_status=st)
        else:
            f = ops.diffattn_grouped_fwd if w.kind == "grouped" else ops.diffattn_fwd
            f(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"], scale=w.scale,
              eps=w.eps, causal=w.causal, dev_status=st)
    torch.cuda.synchronize()
    if st.item() != 0:
        print(f"device status {st.item()}", file=sys.stderr)
        return 1
    print(f"ran {args.iters} x {w.name} (B={w.B})")
    return 0


if __name__ == "__main__":
    sys.exit(main())

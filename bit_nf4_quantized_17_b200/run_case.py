"""Run one QLoRA linear of a workload: quantise, forward, backward.

    python -m bit_nf4_quantized_17_b200.run_case --workload attn_4096 --tokens 4096 --iters 3

A small, self-contained driver for profiling a single kernel configuration
(for example under Nsight Compute with ``-k``/``-c``): it builds the seeded
inputs of one linear of a workload, quantises W once, then runs ``--iters``
forward + backward passes on the current stream and prints the wall time of
the last one.  Times printed here are not benchmark results (use bench.py).
"""

import argparse
import time

import torch

from . import qlora as Q
from . import workloads as WL


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="attn_4096", choices=sorted(WL.WORKLOADS))
    ap.add_argument("--linear", type=int, default=0, help="index of the linear in the layer")
    ap.add_argument("--tokens", type=int, default=None, help="M (default: the workload's first)")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--fwd-only", action="store_true")
    args = ap.parse_args(argv)

    wl = WL.WORKLOADS[args.workload]
    shape = wl.linears[args.linear]
    M = args.tokens if args.tokens is not None else wl.tokens[0]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = WL.linear_inputs(shape, M, 0, dev)
    q = Q.qlora_quantize(inp["W"])
    N, K, r = shape.d_out, shape.d_in, shape.r
    fb, bb = Q.qlora_linear_workspace(M, N, K, r)
    fws = torch.zeros(fb, dtype=torch.uint8, device=dev)
    bws = torch.zeros(bb, dtype=torch.uint8, device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    U = torch.empty((M, r), dtype=torch.float32, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dA = torch.empty((r, K), dtype=torch.float32, device=dev)
    dB = torch.empty((N, r), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    t = 0.0
    for _ in range(args.iters):
        t0 = time.perf_counter()
        Q.qlora_linear_fwd(q, inp["A"], inp["B"], shape.alpha, inp["X"], Y=Y, U_save=U,
                           workspace=fws)
        if not args.fwd_only:
            Q.qlora_linear_bwd(q, inp["A"], inp["B"], shape.alpha, inp["X"], U, inp["dY"],
                               dX=dX, dA=dA, dB=dB, workspace=bws)
        torch.cuda.synchronize()
        t = time.perf_counter() - t0
    Q.qlora_check(fws)
    Q.qlora_check(bws)
    print(f"{args.workload}[{args.linear}] {N}x{K} r={r} M={M}: last iteration {t * 1e6:.1f} us "
          f"(wall clock, not a benchmark)")


if __name__ == "__main__":
    main()

"""Run one entry point of the hot path on a workload's synthetic inputs.

Meant for profilers: it launches the named call a few times on the device and
exits, timing nothing.  For example, from the repository root:

  python -m lora_gemm_b200.cases renoise --workload 2k --launches 3
  python -m lora_gemm_b200.cases euler --workload 2k --launches 3
  python -m lora_gemm_b200.cases lora_linear --workload 2k --layer 2 --tokens 32768

renoise and euler run on the workload's whole latent (the 2K latent is
12,787,200 FP32 elements, 51 MB per tensor); the linear layers on the first
`--tokens` tokens of the layer's activations.  Inputs come from the seeded
recipe in synth.py.
"""

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

import lora_gemm_b200 as lg  # noqa: E402


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("call", choices=["renoise", "euler", "philox_normal", "lora_linear", "lora_linear_mxfp8"])
    ap.add_argument("--workload", default="2k", choices=list(synth.WORKLOADS))
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--layer", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=None)
    args = ap.parse_args(argv)
    w = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sig = [float(torch.tensor(s, dtype=torch.float32)) for s in synth.SIGMA_SCHEDULE]
    if args.call in ("renoise", "euler", "philox_normal"):
        up = synth.upscaled_latent(w, dev)
        x = torch.empty_like(up)
        v = synth.velocity(w, 0, dev)
        for _ in range(args.launches):
            if args.call == "renoise":
                lg.renoise(up, sig[0], w.seed, out=x)
            elif args.call == "euler":
                lg.euler_step(x, v, sig[0], sig[1])
            else:
                lg.philox_normal(up.numel(), w.seed, 0, device=dev)
    else:
        K, N = w.shapes[args.layer]
        M = w.tokens if args.tokens is None else args.tokens
        x = synth.activations(w, K, args.layer, dev, M=M)
        W = synth.weight(w, args.layer, dev)
        As, Bs = synth.adapters(w, args.layer, dev)
        A_cat, B_cat = lg.lora_merge(As, Bs, synth.ADAPTER_SCALES)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        if args.call == "lora_linear":
            for _ in range(args.launches):
                lg.lora_linear(x, W, A_cat, B_cat, y=y)
        else:
            xq, wq = lg.mx_quantize(x), lg.mx_quantize(W)
            for _ in range(args.launches):
                lg.lora_linear_mxfp8(x, xq, wq, A_cat, B_cat, y=y)
    torch.cuda.synchronize()
    status = lg.get_last_device_error()
    if status != lg.LG_OK:
        raise SystemExit(f"device error: {lg.status_string(status)}")
    print(f"{args.call} on {w.name}: {args.launches} launches ok")


if __name__ == "__main__":
    main()

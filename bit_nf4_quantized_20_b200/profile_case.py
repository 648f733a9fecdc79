"""Run one projection of the layer a few times (a small case for profilers).

    python -m bit_nf4_quantized_20_b200.profile_case --proj gate --T 4096 --r 16 --op both --reps 3
    python -m bit_nf4_quantized_20_b200.profile_case --proj all --T 1 --r 64 --s 1 --op fwd --reps 3

Builds the seeded inputs of one Llama-3.1-8B projection (or all seven),
quantizes the weight and calls qlora_linear_fwd / qlora_linear_bwd `reps`
times, printing the CUDA-event time of each call.
"""
from __future__ import annotations

import argparse

import torch

import bit_nf4_quantized_20_b200 as q
from bit_nf4_quantized_20_b200 import inputs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--proj", default="gate", choices=[p[0] for p in inputs.LLAMA8B_PROJ] + ["all"])
    ap.add_argument("--T", type=int, default=4096)
    ap.add_argument("--r", type=int, default=16)
    ap.add_argument("--s", type=float, default=2.0)
    ap.add_argument("--op", default="both", choices=["fwd", "bwd", "both"])
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
    names = [p[0] for p in inputs.LLAMA8B_PROJ]
    dev = torch.device("cuda", 0)
    cases = []
    for i in (range(len(names)) if a.proj == "all" else [names.index(a.proj)]):
        _, N, K = inputs.LLAMA8B_PROJ[i]
        W, X, A, B, dY = inputs.layer_inputs(1, 0, i, a.T, N, K, a.r, device=dev)
        qw = q.quantize_nf4(W)
        del W
        y = torch.empty(a.T, N, dtype=torch.bfloat16, device=dev)
        outs = (torch.empty(a.T, K, dtype=torch.bfloat16, device=dev),
                torch.empty(a.r, K, dtype=torch.bfloat16, device=dev),
                torch.empty(N, a.r, dtype=torch.bfloat16, device=dev))
        cases.append((names[i], N, K, qw, X, A, B, dY, y, outs))
    for rep in range(a.reps):
        for (name, N, K, qw, X, A, B, dY, y, outs) in cases:
            for op in (["fwd", "bwd"] if a.op == "both" else [a.op]):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                if op == "fwd":
                    q.linear_fwd(X, qw, A, B, a.s, out=y)
                    fl = 2.0 * a.T * N * K + 2.0 * a.T * a.r * (N + K)
                else:
                    q.linear_bwd(dY, X, qw, A, B, a.s, outs=outs)
                    fl = 2.0 * a.T * N * K + 4.0 * a.T * a.r * (N + K)
                e1.record()
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1)
                print(f"{name} T={a.T} {op} rep {rep}: {ms:.4f} ms  {fl / ms / 1e9:.1f} TFLOP/s", flush=True)
    q.get_error(dev)


if __name__ == "__main__":
    main()

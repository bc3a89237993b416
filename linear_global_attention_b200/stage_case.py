"""Run one stage of the library on random bf16 inputs and print its kernel times.

    python -m linear_global_attention_b200.stage_case --stage sparse --views 384 --heads 1
    python -m linear_global_attention_b200.stage_case --stage linear --views 128 --heads 16
    python -m linear_global_attention_b200.stage_case --stage affine --views 128 --heads 16

A small, self-contained case for profilers: inputs are generated on the GPU
(torch.randn), the stage runs `--warmup` times, then `--reps` times with the
library's kernel event records on, and one JSON line reports mean milliseconds
per launch of each kernel. For the sparse stage it also reports the kept-tile
TFLOP/s (4*d FLOPs per visible logit); for the linear stage the HBM GB/s of its
compulsory bytes (Q, K, V read once, O written once). The linear stage reads
Q/K/V as strided slices of one [N, 3*H*64] projection buffer, as the stacked
layer does. The affine stage accumulates the fit moments of random x, y
([N, H, 64] bf16) and solves the pooled fit; it reports the float64 TFLOP/s of
the moments pass (2 * 2 * 64 * 64 FLOPs per (token, head): x x^T and x y^T)
and the GB/s of its input bytes.
"""
from __future__ import annotations

import argparse
import json

import torch

import linear_global_attention_b200 as zb


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--stage", choices=["sparse", "linear", "affine"], default="sparse")
    ap.add_argument("--views", type=int, default=512)
    ap.add_argument("--grid", type=int, default=37)
    ap.add_argument("--heads", type=int, default=4)
    ap.add_argument("--y", type=float, default=0.8)
    ap.add_argument("--warmup", type=int, default=1)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
    H = a.heads
    g = zb.geom(a.views, a.grid, a.grid, H)
    N = g.n_tokens
    gen = torch.Generator(device="cuda").manual_seed(1)
    if a.stage == "sparse":
        q, k, v = (torch.randn((N, H, 64), generator=gen, device="cuda").to(torch.bfloat16) for _ in range(3))
        ws = zb.workspace(g, zb.ZEBRA_OP_SPARSE, zb.ZEBRA_BF16, a.y)

        def run(out):
            zb.zebra_sparse_attn(g, q, k, v, a.y, out, ws)
    elif a.stage == "affine":
        x, y = (torch.randn((N, H, 64), generator=gen, device="cuda").to(torch.bfloat16) for _ in range(2))
        ws = zb.workspace(g, zb.ZEBRA_OP_AFFINE)
        mom = zb.affine_moments_buffer(g)
        A = torch.empty((H, 64, 64), device="cuda")
        b = torch.empty((H, 64), device="cuda")

        def run(out):
            mom.zero_()
            zb.zebra_affine_moments(g, x, y, mom, ws)
            zb.zebra_affine_solve(g, mom, 1e-3, A, b)
    else:
        qkv = torch.randn((N, 3 * H * 64), generator=gen, device="cuda").to(torch.bfloat16)
        q, k, v = (qkv[:, i * H * 64:(i + 1) * H * 64].view(N, H, 64) for i in range(3))
        ws = zb.workspace(g, zb.ZEBRA_OP_LINEAR)

        def run(out):
            zb.zebra_linear_attn(g, q, k, v, None, None, out, ws)
    out = torch.empty((N, H, 64), device="cuda", dtype=torch.bfloat16)
    for _ in range(a.warmup):
        run(out)
    torch.cuda.synchronize()
    zb.zebra_profile_enable(True)
    for _ in range(a.reps):
        run(out)
    rep = zb.zebra_profile_report()
    zb.zebra_profile_enable(False)
    if zb.zebra_sync_status() != zb.ZEBRA_OK:
        raise SystemExit(zb.zebra_last_error())
    ks = {n: round(ms / c, 4) for n, (c, ms) in rep["kernels"].items()}
    res = {"stage": a.stage, "views": a.views, "grid": a.grid, "heads": H, "tokens": N, "kernels_ms": ks}
    if a.stage == "sparse":
        n, ms = rep["kernels"]["attn_sparse_rows"]
        logits = rep["logits"]["sparse_rows"] / n
        res.update(y=a.y, logits_per_launch=logits, tflops=round(256 * logits / (ms / n / 1e3) / 1e12, 2))
    elif a.stage == "affine":
        n, ms = rep["kernels"]["affine_moments"]
        t = ms / n / 1e3
        res.update(fp64_tflops=round(4 * 64 * 64 * N * H / t / 1e12, 3), gbs=round(2 * N * H * 64 * 2 / t / 1e9, 1))
    else:
        ms = sum(rep["kernels"][x][1] for x in ("linear_state", "linear_reduce", "linear_apply")) / a.reps
        res.update(ms=round(ms, 4), gbs=round(8 * N * H * 64 / (ms / 1e3) / 1e9, 1))
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()

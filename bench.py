#!/usr/bin/env python
"""Benchmark of the Zebra3D hybrid global-attention stack on B200.

Workload (the configuration the headline metric is quoted on): 1,024 views of
a 37x37 patch grid plus 5 special tokens each (N = 1,406,976 tokens), model
dim 1024, 16 heads of 64, 24 stacked global-attention layers allocated 0.7L/0.8S
(layers 0-16 linear, 17-23 tile-sparse at y = 0.8), bf16, random-init
projections ~ N(0, 0.02^2) and x0 ~ N(0, 1) from seed 4.

One step = one pass of the whole stack (every step of the hot path: projections,
pooling/packing, selection, sparse attention, dense special rows, linear
state/apply, residual) over x0. Metric: tokens/s per layer = n_gpus * N * 24 /
(device time of one step). Each step also copies x0 host->device before and
x24 device->host after the stack inside the e2e timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl zebra|reference]

--impl reference times the CPU oracle (fp64 NumPy, this repository's test
oracle) on bounded samples of the same workload, extrapolated to a full step.
Multi-GPU (torchrun): every rank runs its own replica (weak scaling); times
are the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "global-attn tokens/s per layer at 1,024 views (sparse, linear, hybrid) + % roofline"
UNIT = "tokens/s"
WORKLOAD = "stack_v1024"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["zebra", "reference"], default="zebra")
    p.add_argument("--views", type=int, default=None, help="override the view count (quick runs only)")
    p.add_argument("--no-dense", action="store_true", help="skip the dense softmax baseline")
    p.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    p.add_argument("--no-scaling", action="store_true",
                   help="skip the view-scaling workloads and the other operating points")
    p.add_argument("--json-extra", default=None, help="also write the full result dict to this file")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
# DRAM traffic of the sparse attention kernel, from an ncu capture of
# dram__bytes_read.sum + dram__bytes_write.sum over every launch of one call
# at 1,024 views x 1 head: bytes per (head, query tile) work item.
# Valid only for the kernel sources it was taken on; otherwise traffic is null.
SPARSE_TRAFFIC = {"bytes_per_item": 672131, "sources_sha1": "012db3d21873ee1f105e9169eafbf2ac030aa919"}
SPARSE_SOURCES = ("linear_global_attention_b200/csrc/attn_tc.cuh", "linear_global_attention_b200/csrc/attn.cu",
                  "linear_global_attention_b200/csrc/tc_prims.cuh")


def sparse_sources_sha1() -> str:
    import hashlib
    h = hashlib.sha1()
    for rel in SPARSE_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def sparse_traffic_per_launch(items_per_launch: float):
    """Measured DRAM bytes per launch of the sparse kernel, or None when not measured for these sources."""
    t = SPARSE_TRAFFIC
    if t["bytes_per_item"] is None or t["sources_sha1"] != sparse_sources_sha1():
        return None
    return round(t["bytes_per_item"] * items_per_launch)


def stage_rates(kern: dict, g, hbm_gbs: float) -> dict:
    """Rates of the smaller sparse-stage kernels per sparse layer, from their event times.

    kern: {name: (records, total_ms)} of the profile report; g: the layer
    geometry (bf16). pool_pack: algorithmic bytes = patch rows of Q, K, V read
    once; packed Q tiles [H, T, 64, 64], K and V in the dense layout of 8-row
    groups (H x views x rows-per-view rows), fp32 means and landmark rows
    written.
    tile_scores: 2 * 64 FLOPs per (query tile, key tile) score (the rate of fp32
    scores it delivers; it computes them as one bf16 tensor-core GEMM with
    K = 6 x 64 over the means' bf16 parts, 2 * 384 FLOPs per score).
    tile_select: the T x T fp32 scores read once per head.
    """
    layers = kern.get("pool_pack", (0, 0.0))[0]
    if not layers:
        return {}
    H, T = g.heads, g.n_tiles
    t_pad = (T + 63) // 64 * 64
    patches = g.views * g.grid_h * g.grid_w
    out = {}
    ms = kern["pool_pack"][1] / layers
    tr, tc = (g.grid_h + 7) // 8, (g.grid_w + 7) // 8
    rl, cl = g.grid_h - 8 * (tr - 1), g.grid_w - 8 * (tc - 1)
    rows_per_view = 8 * g.grid_w * (tr - 1) + rl * 8 * (tc - 1) + (rl * cl + 7) // 8 * 8
    nbytes = (3 * patches * H * 128 + H * T * 64 * 128 + 2 * H * g.views * rows_per_view * 128
              + 3 * H * T * 64 * 4 + 2 * H * t_pad * 128)
    gbs = nbytes / (ms / 1e3) / 1e9
    out["pool_pack"] = {"ms_per_layer": round(ms, 3), "bytes_per_layer": nbytes, "gbs": round(gbs, 1),
                        "frac_hbm": round(gbs / hbm_gbs, 4)}
    if "tile_scores" in kern:
        ms = kern["tile_scores"][1] / layers
        out["tile_scores"] = {"ms_per_layer": round(ms, 3),
                              "fp32_score_tflops": round(2 * 64 * T * T * H / (ms / 1e3) / 1e12, 2),
                              "bf16_gemm_tflops": round(2 * 384 * T * T * H / (ms / 1e3) / 1e12, 1)}
    if "tile_select" in kern:
        ms = kern["tile_select"][1] / layers
        out["tile_select"] = {"ms_per_layer": round(ms, 3), "score_gbs": round(4 * T * T * H / (ms / 1e3) / 1e9, 1)}
    return out


def dist_setup():
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=900))
    else:
        torch.cuda.set_device(0)
    return ws, rank, local


def max_over_ranks(x: float, ws: int) -> float:
    """Max of a per-rank float over all ranks (all-reduce on the process group's device)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int):
    import torch
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        ident = str(device_index)
        try:
            import torch
            ident = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            pass
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-i", ident, "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(5)
            except subprocess.TimeoutExpired:
                self.p.kill()
        self.f.flush()
        rows = []
        with open(self.f.name) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) == 7:
                    rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = [n for i, n in enumerate(names) if any(r[3 + i] == "Active" for r in rows)]
        loaded = [x for x in sm if x > 500] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": float(rows[0][1]) if rows[0][1].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_zebra(args):
    import numpy as np
    import torch

    import linear_global_attention_b200 as zb
    import synth

    ws_n, rank, local = dist_setup()
    w = synth.WORKLOADS[WORKLOAD]
    if args.views:
        import dataclasses
        w = dataclasses.replace(w, views=args.views)
    V, Hp, Wp, H, D = w.views, w.grid_h, w.grid_w, w.heads, w.model_dim
    g = zb.geom(V, Hp, Wp, H)
    N, L = g.n_tokens, w.layers
    kinds = synth.stack_layer_kinds(w)
    y = w.y[0]

    # inputs: x0 in pinned host memory; weights resident on the device
    t0 = time.time()
    x0_host = torch.from_numpy(synth.stack_x0(w)).to(torch.bfloat16).pin_memory()
    wq, wo, As, bs = [], [], [], []
    for layer in range(L):
        a, b = synth.stack_layer_weights(w, layer)
        wq.append(torch.from_numpy(a).to(torch.bfloat16).cuda())
        wo.append(torch.from_numpy(b).to(torch.bfloat16).cuda())
        if kinds[layer] == "linear":
            A, bb = synth.affine(H, w.seed, layer)
            As.append(torch.from_numpy(A).cuda())
            bs.append(torch.from_numpy(bb).cuda())
        else:
            As.append(None)
            bs.append(None)
    gen_s = time.time() - t0
    wsb = max(zb.zebra_workspace_bytes(g, zb.ZEBRA_OP_HYBRID_LINEAR, zb.ZEBRA_BF16, y),
              zb.zebra_workspace_bytes(g, zb.ZEBRA_OP_HYBRID_SPARSE, zb.ZEBRA_BF16, y))
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    x0 = torch.empty((N, D), dtype=torch.bfloat16, device="cuda")
    xa = torch.empty_like(x0)
    xb = torch.empty_like(x0)
    out_host = torch.empty((N, D), dtype=torch.bfloat16).pin_memory()
    kind_id = {"linear": zb.ZEBRA_LAYER_LINEAR, "sparse": zb.ZEBRA_LAYER_SPARSE}

    def stack(layer_events=None):
        src = x0
        for layer in range(L):
            dst = xa if layer % 2 == 0 else xb
            zb.zebra_hybrid_layer(g, kind_id[kinds[layer]], src, wq[layer], wo[layer], As[layer], bs[layer], y, dst,
                                  ws)
            if layer_events is not None:
                layer_events[layer].record()
            src = dst
        return src

    def step(ev):
        # ev: [e2e start, stack start, per-layer..., stack end(=last layer), e2e end]
        ev[0].record()
        x0.copy_(x0_host, non_blocking=True)
        ev[1].record()
        res = stack(ev[2:2 + L])
        out_host.copy_(res, non_blocking=True)
        ev[2 + L].record()

    def new_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(L + 3)]

    for _ in range(args.warmup):
        step(new_events())
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    barrier(ws_n)

    clocks = ClockSampler(torch.cuda.current_device())
    zb.zebra_profile_enable(True)
    launches0 = zb.zebra_launch_count()
    evs = [new_events() for _ in range(args.steps)]
    barrier(ws_n)
    for i in range(args.steps):
        step(evs[i])
    barrier(ws_n)
    launches = zb.zebra_launch_count() - launches0
    clk = clocks.stop()
    prof = zb.zebra_profile_report()
    zb.zebra_profile_enable(False)
    assert zb.zebra_sync_status() == zb.ZEBRA_OK

    dev_ms = sum(e[1].elapsed_time(e[1 + L]) for e in evs)
    e2e_ms = sum(e[0].elapsed_time(e[2 + L]) for e in evs)
    per_layer = {"linear": [], "sparse": []}
    for e in evs:
        prev = e[1]
        for layer in range(L):
            per_layer[kinds[layer]].append(prev.elapsed_time(e[2 + layer]))
            prev = e[2 + layer]
    dev_ms = max_over_ranks(dev_ms, ws_n)
    e2e_ms = max_over_ranks(e2e_ms, ws_n)
    ms_step = dev_ms / args.steps
    value = ws_n * N * L / (ms_step / 1e3)
    e2e_value = ws_n * N * L / (e2e_ms / args.steps / 1e3)

    # roofline of the dominant kernel
    pk = peaks()
    kern = prof["kernels"]
    dom = max(kern.items(), key=lambda kv: kv[1][1])
    sparse_calls, sparse_ms = kern.get("attn_sparse_rows", (0, 0.0))
    sparse_launches = max(prof["launches"].get("attn_sparse_rows", 0), 1)
    sparse_flops = 4 * 64 * prof["logits"].get("sparse_rows", 0)
    achieved = sparse_flops / (sparse_ms / 1e3) / 1e12 if sparse_ms else 0.0
    items_per_launch = H * g.n_tiles * max(sparse_calls, 1) / sparse_launches
    roofline = {"kernel": "attn_sparse_rows (attn_tc_kernel)", "bound": "tensor", "achieved": round(achieved, 2),
                "peak": pk["bf16_sustained"], "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_sustained"], 4),
                "traffic": sparse_traffic_per_launch(items_per_launch),
                "peak_source": f"{pk['source']} bf16 sustained",
                "algorithmic_flops_per_launch": sparse_flops / sparse_launches,
                "avg_launch_ms": sparse_ms / sparse_launches,
                "launches_per_call": sparse_launches / max(sparse_calls, 1),
                "work_items_per_launch": round(items_per_launch, 1),
                # a 64-row query tile gives M = 64 MMAs, which use half of the tensor datapath
                # (measured issue rate of M = 64 tcgen05.mma on this part): context, not the peak
                "frac_of_m64_ceiling": round(achieved / (pk["bf16_sustained"] / 2), 4)}
    # linear stage: compulsory HBM bytes (Q, K, V read once, O written once, bf16)
    lin_bytes = 8 * N * H * 64
    lin_ms = sum(kern.get(n, (0, 0.0))[1] for n in ("linear_state", "linear_reduce", "linear_apply"))
    lin_layers = max(kern.get("linear_state", (0, 0))[0], 1)
    lin_gbs = lin_bytes / (lin_ms / lin_layers / 1e3) / 1e9 if lin_ms else 0.0
    stages = {name: {"launches": n, "total_ms": round(ms, 3), "share": round(ms / sum(v[1] for v in kern.values()), 4)}
              for name, (n, ms) in kern.items()}

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": ws_n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded x0 ~ N(0,1), W ~ N(0,0.02^2))",
        "config": {"workload": f"{WORKLOAD}: {V} views x (37x37 patches + 5 special) = {N:,} tokens, "
                               f"{L} layers 0.7L/0.8S (17 linear + 7 tile-sparse y=0.8), dim 1024, 16 heads x 64",
                   "views": V, "tokens": N, "layers": L, "allocation": "0.7L/0.8S", "parallelism": f"replica x{ws_n}",
                   "l2": "inputs larger than L2 (x0 = %.2f GB bf16)" % (N * D * 2 / 1e9)},
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": N * D * 2,
                "d2h_bytes_per_step": N * D * 2},
        "gpu_launches": int(launches),
        "clocks": clk,
        "layer_ms": {k: round(statistics.mean(v), 3) for k, v in per_layer.items() if v},
        "linear_stage_hbm": {"gbs": round(lin_gbs, 1), "peak_gbs": pk["hbm_gbs"],
                             "frac": round(lin_gbs / pk["hbm_gbs"], 4), "compulsory_bytes": lin_bytes},
        "sparse_prep": stage_rates(kern, g, pk["hbm_gbs"]),
        "kernels": stages,
        "dominant_kernel": dom[0],
        "input_gen_s": round(gen_s, 1),
    }

    # the other operating points of the page (xL/yS), from measured per-layer
    # times: one extra C4 sparse layer at y = 0.6 is timed here
    if rank == 0 and not args.no_scaling:
        first_sparse = kinds.index("sparse")
        f = lambda: zb.zebra_hybrid_layer(g, zb.ZEBRA_LAYER_SPARSE, x0, wq[first_sparse], wo[first_sparse], None,
                                          None, 0.6, xa, ws)
        sp06_ms, sp06_all = timed_ms(f, 2, warmup=0)
        t_lin = statistics.mean(per_layer["linear"])
        t_sp08 = statistics.mean(per_layer["sparse"])
        layer_ms = {"0.8": t_sp08, "0.6": sp06_ms}
        ops = {}
        for name, lin_frac, yy in (("0.5L/0.6S", 0.5, "0.6"), ("0.5L/0.8S", 0.5, "0.8"), ("0.7L/0.6S", 0.7, "0.6"),
                                   ("0.7L/0.8S", 0.7, "0.8")):
            n_lin = int(math.floor(lin_frac * L + 0.5))
            st_ms = ms_step if name == "0.7L/0.8S" else n_lin * t_lin + (L - n_lin) * layer_ms[yy]
            ops[name] = {"linear_layers": n_lin, "sparse_layers": L - n_lin, "stack_ms": round(st_ms, 1),
                         "tokens_per_s_per_layer": round(ws_n * N * L / (st_ms / 1e3), 1),
                         "source": "measured step" if name == "0.7L/0.8S" else "sum of measured per-layer times"}
        result["operating_points"] = {"sparse_layer_ms_y0.6": round(sp06_ms, 1),
                                      "sparse_layer_ms_y0.6_reps": [round(x, 1) for x in sp06_all],
                                      "sparse_layer_ms_y0.8": round(t_sp08, 1), "linear_layer_ms": round(t_lin, 2),
                                      "points": ops}
    if not args.no_dense and rank == 0:
        result["dense_baseline"] = dense_baseline(g, N, H, D, kern, ms_step, L)
        if "operating_points" in result:
            for v in result["operating_points"]["points"].values():
                v["speedup_vs_dense_stack"] = round(result["dense_baseline"]["stack_ms"] / v["stack_ms"], 3)
    if rank == 0 and not args.no_scaling:
        del ws
        import torch
        torch.cuda.empty_cache()
        result["view_scaling"] = view_scaling(pk)
    if not args.no_cpu and rank == 0:
        result["cpu_baseline"] = cpu_baseline(w, budget_s=20.0)
    if ws_n > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return result, rank


def timed_ms(fn, reps: int, warmup: int = 1):
    """Median device time (CUDA events on the current stream) of `reps` calls of fn after `warmup` calls."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    out = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1))
    return statistics.median(out), out


def sdpa_ms(q, k, v, reps: int = 3):
    """Median time of torch SDPA (bf16, flash/cuDNN) over [1, H, N, 64] tensors."""
    import torch
    f = lambda: torch.nn.functional.scaled_dot_product_attention(q, k, v)
    torch.nn.functional.scaled_dot_product_attention(q[:, :, :65536], k[:, :, :65536], v[:, :, :65536])
    return timed_ms(f, reps, warmup=0)


def view_scaling(pk, reps: int = 10):
    """The view-scaling workloads at 1 GPU (section "Speedup scales with the number of
    input views"), each timed as whole stage calls (pooling/packing, selection,
    attention, special rows; or the three linear kernels) with CUDA events:
      sparse_v32       32 views x (32x32 + 5), 16 heads, y = 0.8, latent recipe;
      linear_v128      128 views x (37x37 + 5), 16 heads, the full linear stage;
      sidebyside_v512  512 views x (37x37 + 5), 16 heads, y = 0.6 and y = 0.8,
                       latent recipe, against torch SDPA on identical inputs and
                       against the library's own dense path (y = 0).
    Median of `reps` calls (3 for the 512-view calls and SDPA)."""
    import torch

    import linear_global_attention_b200 as zb
    import synth

    def inputs(name):
        w = synth.WORKLOADS[name]
        g = zb.geom(w.views, w.grid_h, w.grid_w, w.heads)
        q, k, v = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in synth.qkv(w))
        desc = (f"{name}: {w.views} views x ({w.grid_h}x{w.grid_w} patches + 5 special) = {g.n_tokens:,} tokens, "
                f"{w.heads} heads x 64, bf16, {w.recipe} recipe, seed {w.seed}")
        return w, g, q, k, v, desc

    def sparse(g, q, k, v, y, n):
        ws = zb.workspace(g, zb.ZEBRA_OP_SPARSE, zb.ZEBRA_BF16, y)
        o = torch.empty_like(q)
        f = lambda: zb.zebra_sparse_attn(g, q, k, v, y, o, ws)
        f()
        zb.zebra_profile_enable(True)
        ms, all_ms = timed_ms(f, n, warmup=0)
        rep = zb.zebra_profile_report()
        zb.zebra_profile_enable(False)
        calls, att_ms = rep["kernels"]["attn_sparse_rows"]
        tfl = 256 * rep["logits"]["sparse_rows"] / (att_ms / 1e3) / 1e12
        del ws, o
        res = {"keep": zb.zebra_keep_count(y, g.n_tiles), "ms": round(ms, 3), "ms_reps": [round(x, 3) for x in all_ms],
               "tokens_per_s": round(g.n_tokens / (ms / 1e3), 1), "attn_kernel_ms": round(att_ms / calls, 3),
               "attn_kernel_tflops": round(tfl, 1), "attn_frac_of_sustained_bf16": round(tfl / pk["bf16_sustained"], 4)}
        if y > 0:
            # near-ties of the same selection (the keep-th and next score within a
            # relative 1e-5), as the selector flags them (outside the timing)
            qm = torch.empty(g.heads, g.n_tiles, 64, device="cuda")
            km = torch.empty_like(qm)
            zb.zebra_tile_pool(g, q, qm)
            zb.zebra_tile_pool(g, k, km)
            mask = torch.empty(g.heads, g.n_tiles, g.mask_words, dtype=torch.int32, device="cuda")
            near = torch.empty(g.heads, g.n_tiles, dtype=torch.uint8, device="cuda")
            wss = zb.workspace(g, zb.ZEBRA_OP_SELECT, zb.ZEBRA_BF16, y)
            zb.zebra_tile_select(g, qm, km, y, mask, near, wss)
            res["near_tie_rows"] = {"count": int(near.sum().item()), "of": g.heads * g.n_tiles}
            del qm, km, mask, near, wss
        return res

    out = {}
    w, g, q, k, v, desc = inputs("sparse_v32")
    out["sparse_v32"] = {"workload": desc, "y=0.8": sparse(g, q, k, v, 0.8, reps)}
    del q, k, v
    w, g, q, k, v, desc = inputs("linear_v128")
    A, b = (torch.from_numpy(x).cuda() for x in synth.affine(w.heads, w.seed))
    ws = zb.workspace(g, zb.ZEBRA_OP_LINEAR)
    o = torch.empty_like(q)
    ms, all_ms = timed_ms(lambda: zb.zebra_linear_attn(g, q, k, v, A, b, o, ws), 2 * reps, warmup=3)
    nbytes = 8 * g.n_tokens * g.heads * 64
    out["linear_v128"] = {"workload": desc, "ms": round(ms, 4), "tokens_per_s": round(g.n_tokens / (ms / 1e3), 1),
                          "compulsory_bytes": nbytes, "gbs": round(nbytes / (ms / 1e3) / 1e9, 1),
                          "frac_of_measured_hbm": round(nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"], 4)}
    del q, k, v, ws, o
    w, g, q, k, v, desc = inputs("sidebyside_v512")
    res = {"workload": desc}
    for y in (0.6, 0.8):
        res[f"y={y}"] = sparse(g, q, k, v, y, 3)
    # the library's own dense path: y = 0 keeps every tile (one call)
    res["own_dense_y=0"] = sparse(g, q, k, v, 0.0, 1)
    qt, kt, vt = (x.permute(1, 0, 2).unsqueeze(0).contiguous() for x in (q, k, v))   # [1, H, N, 64]
    del q, k, v
    med, all_ms = sdpa_ms(qt, kt, vt, reps=3)
    N, H = g.n_tokens, g.heads
    res["sdpa"] = {"ms": round(med, 1), "ms_reps": [round(x, 1) for x in all_ms],
                   "tflops": round(4 * 64 * N * N * H / (med / 1e3) / 1e12, 1)}
    for key in ("y=0.6", "y=0.8", "own_dense_y=0"):
        res[key]["speedup_vs_sdpa"] = round(med / res[key]["ms"], 3)
    out["sidebyside_v512"] = res
    del qt, kt, vt
    torch.cuda.empty_cache()
    return out


def dense_baseline(g, N, H, D, kern, ms_step, L):
    """Same-GPU dense softmax layer on identical shapes: torch SDPA (flash/cuDNN,
    bf16) over [1, 16, N, 64] (median of 3 calls) plus this run's projection
    GEMM time per layer."""
    import torch
    gen = torch.Generator(device="cuda").manual_seed(0)
    q = torch.randn((1, H, N, 64), device="cuda", dtype=torch.bfloat16, generator=gen)
    k = torch.randn_like(q)
    v = torch.randn_like(q)
    sdpa_ms_med, sdpa_all = sdpa_ms(q, k, v, reps=3)
    sdpa_ms_ = sdpa_ms_med
    del q, k, v
    gemm_n, gemm_ms = kern.get("cublasLt_gemm", (0, 0.0))
    gemm_per_layer = gemm_ms / max(gemm_n, 1) * 2
    layer_ms = sdpa_ms_ + gemm_per_layer
    flops = 4 * 64 * N * N * H
    return {"impl": "torch.nn.functional.scaled_dot_product_attention (bf16) + the stack's projection GEMMs",
            "sdpa_ms": round(sdpa_ms_, 1), "sdpa_ms_reps": [round(x, 1) for x in sdpa_all],
            "sdpa_tflops": round(flops / (sdpa_ms_ / 1e3) / 1e12, 1),
            "layer_ms": round(layer_ms, 1), "stack_ms": round(layer_ms * L, 1),
            "tokens_per_s_per_layer": round(N / (layer_ms / 1e3), 1),
            "hybrid_speedup": round(layer_ms * L / ms_step, 3)}


# ---------------------------------------------------------------------------
# CPU oracle (the reference arm and the cpu_baseline)
# ---------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return None


def cpu_baseline(w, budget_s=20.0, sample_tiles=4):
    """The fp64 oracle on a bounded sample of one step, extrapolated to a step.

    Sample (one head): the sparse stage for `sample_tiles` query tiles at the
    full 1,024-view geometry (tile pooling, selection over all tiles, kept
    tokens, landmarks, special keys), with iid N(0,1) Q/K/V; the linear stage
    on a 1/8-size geometry (128 views), whose cost is linear in the token count;
    the projections of 4,096 rows. The sparse call is timed once more without
    query tiles (its pooling and setup); the difference is the sample tiles'
    cost. Extrapolation: x8 for the linear stage, x(T / sample_tiles) for the
    sparse tiles, x16 heads, x(N / 4,096) rows, then 17 linear + 7 sparse
    layers.
    """
    import dataclasses

    import numpy as np

    import oracle
    import synth

    g = oracle.Geom(w.views, w.grid_h, w.grid_w, 1)
    N, T = g.n_tokens, g.n_tiles
    scale = 8
    gs = oracle.Geom(max(1, w.views // scale), w.grid_h, w.grid_w, 1)
    ratio = N / gs.n_tokens
    q, k, v = (synth.normal_blocks((1, 64), N, 777, i) for i in range(3))
    qs, ks, vs = (x[:gs.n_tokens] for x in (q, k, v))
    A, b = synth.affine(1, 777)
    keep = oracle.keep_count(w.y[0], T)
    rng = np.random.default_rng(0)
    tiles = np.sort(rng.choice(T, sample_tiles, replace=False))
    t0 = time.perf_counter()
    oracle.linear_stage(qs, ks, vs, gs, A, b)
    t_lin = (time.perf_counter() - t0) * ratio
    # the call pools every tile before its query tiles: time it once without
    # query tiles too, and take the query tiles' share as the difference
    none = np.zeros(0, np.int64)
    t0 = time.perf_counter()
    oracle.sparse_stage(q, k, v, g, keep, query_tiles=none, special_rows=none)
    t_base = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.sparse_stage(q, k, v, g, keep, query_tiles=tiles, special_rows=none)
    t_call = time.perf_counter() - t0
    t_tiles = max(t_call - t_base, 1e-9)
    rows = 4096
    xs = rng.standard_normal((rows, w.model_dim))
    wqkv = rng.standard_normal((3 * w.model_dim, w.model_dim))
    wo = rng.standard_normal((w.model_dim, w.model_dim))
    t0 = time.perf_counter()
    xs @ wqkv.T
    xs @ wo.T
    t_proj = (time.perf_counter() - t0) * N / rows
    H = w.heads
    sparse_layer = H * (t_base + T / sample_tiles * t_tiles)
    linear_layer = H * t_lin
    n_lin = w.n_linear
    step_s = n_lin * (linear_layer + t_proj) + (w.layers - n_lin) * (sparse_layer + t_proj)
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count()
    return {"value": round(N * w.layers / step_s, 3), "unit": UNIT, "cores": cores, "blas_threads": _blas_threads(),
            "kind": "oracle",
            "sample": f"1 head: {sample_tiles} sparse query tiles at the full {w.views}-view geometry (its tile "
                      f"pooling timed apart), the linear stage on {gs.views} views (x{ratio:.0f}), projections of "
                      f"{rows} rows; "
                      f"extrapolated to 16 heads, all {T} tiles and the 24-layer step",
            "step_s_extrapolated": round(step_s, 1),
            "measured_s": {"sparse_call": round(t_call, 2), "sparse_call_no_query_tiles": round(t_base, 2),
                           "linear_head_scaled": round(t_lin, 2),
                           "proj": round(t_proj, 2)}}


def run_reference(args):
    import synth
    rank = int(os.environ.get("RANK", "0"))
    ws_n = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return None, rank
    w = synth.WORKLOADS[WORKLOAD]
    if args.views:
        import dataclasses
        w = dataclasses.replace(w, views=args.views)
    for _ in range(args.warmup):
        cpu_baseline(w, sample_tiles=1)
    vals = []
    last = None
    for _ in range(args.steps):
        last = cpu_baseline(w)
        vals.append(last["value"])
    value = statistics.mean(vals)
    N = w.n_tokens
    res = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws_n, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(N * w.layers / value * 1e3, 1), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": f"{WORKLOAD}: {w.views} views, {N:,} tokens, {w.layers} layers 0.7L/0.8S"},
           "impl": "reference",
           "cpu_baseline": {"kind": "oracle", "cores": last["cores"], "sample": last["sample"], "value": value},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return res, rank


def main():
    args = parse()
    if args.impl == "reference":
        res, rank = run_reference(args)
    else:
        res, rank = run_zebra(args)
    if rank == 0 and res is not None:
        line = json.dumps(res)
        print(line, flush=True)
        if args.json_extra:
            with open(args.json_extra, "w") as f:
                f.write(json.dumps(res, indent=1))


if __name__ == "__main__":
    main()

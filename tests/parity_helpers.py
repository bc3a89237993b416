"""Helpers of the GPU parity tests: run the C ABI on seeded inputs and compare
with the fp64 oracle.

Tolerances:
  bf16 inputs, fp32 accumulation: max |err| <= 2e-2 and relative L2 <= 5e-3
    against the fp64 oracle (the acceptance bar stated for the method's
    outputs);
  fp32 inputs: max |err| <= 2e-4 and relative L2 <= 2e-5, derived from fp32
    arithmetic (unit roundoff 6e-8) through softmax logits of magnitude up to
    ~60 on the tiny workload (exp amplifies an absolute logit error e into a
    relative weight error e; e ~ 60 * 64 * 6e-8 ~ 2e-4 worst case).
Selections are compared bit for bit except on rows whose keep-th and
(keep+1)-th oracle scores lie within a relative gap of 1e-5 (near-ties); those
rows are counted, the GPU's choice is checked to be a valid top-k under that
gap, and their outputs are left out of the element-wise comparison.
"""
from __future__ import annotations

import numpy as np
import torch

import linear_global_attention_b200 as zb
import oracle

TOL = {"bf16": (2e-2, 5e-3), "f32": (2e-4, 2e-5)}


def dev(x: np.ndarray, dtype: str):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.cuda()


def host(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def zgeom(g: oracle.Geom):
    return zb.geom(g.views, g.grid_h, g.grid_w, g.heads, n_special=g.n_special)


def unpack_mask(mask_t, T: int) -> np.ndarray:
    m = mask_t.cpu().numpy().astype("<u4")
    bits = np.unpackbits(m.view(np.uint8), axis=-1, bitorder="little")
    return bits[..., :T].astype(bool)


def errors(got: np.ndarray, want: np.ndarray):
    d = got - want
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(want), 1e-30)) if d.size else 0.0
    return max_abs, rel


# (label, dtype, max_abs, rel_l2) of every comparison in this session, printed by
# the terminal-summary hook in conftest.py
RECORD = []
# (label, query-tile rows compared, rows with an oracle near-tie) of every
# selection comparison, printed by the same hook
NEAR_TIES = []


def record_near_ties(what: str, rows: int, near: int):
    NEAR_TIES.append((what, int(rows), int(near)))


def assert_close(got, want, dtype: str, what: str = ""):
    max_abs, rel = errors(got, want)
    ta, tr = TOL[dtype]
    RECORD.append((what, dtype, float(max_abs), float(rel)))
    assert max_abs <= ta and rel <= tr, f"{what}: max_abs {max_abs:.3e} (tol {ta}), rel_l2 {rel:.3e} (tol {tr})"
    return max_abs, rel


def run_sparse(g: oracle.Geom, q, k, v, y: float, dtype: str, mask=None):
    zg = zgeom(g)
    qd, kd, vd = dev(q, dtype), dev(k, dtype), dev(v, dtype)
    out = torch.empty_like(qd)
    ws = zb.workspace(zg, zb.ZEBRA_OP_SPARSE, zb.ZEBRA_BF16 if dtype == "bf16" else zb.ZEBRA_F32, y)
    zb.zebra_sparse_attn(zg, qd, kd, vd, y, out, ws, mask=mask)
    torch.cuda.synchronize()
    return out


def run_select(g: oracle.Geom, q, k, y: float, dtype: str):
    """GPU tile means (pool) + selection; returns (mask bool [H,T,T], near_tie [H,T], keep, qm, km)."""
    zg = zgeom(g)
    T, W = zg.n_tiles, zg.mask_words
    qm = torch.empty(g.heads, T, 64, device="cuda")
    km = torch.empty_like(qm)
    zb.zebra_tile_pool(zg, dev(q, dtype), qm)
    zb.zebra_tile_pool(zg, dev(k, dtype), km)
    mask = torch.empty(g.heads, T, W, dtype=torch.int32, device="cuda")
    nt = torch.empty(g.heads, T, dtype=torch.uint8, device="cuda")
    ws = zb.workspace(zg, zb.ZEBRA_OP_SELECT, zb.ZEBRA_BF16, y)
    keep = zb.zebra_tile_select(zg, qm, km, y, mask, nt, ws)
    torch.cuda.synchronize()
    return unpack_mask(mask, T), nt.cpu().numpy().astype(bool), keep, mask


def check_selection(g: oracle.Geom, q, k, keep: int, gpu_sel: np.ndarray, heads=None, rows=None, what=None):
    """Bit-exact selection outside oracle near-ties; valid top-k inside them.
    Returns {h: near-tie rows (oracle)}; the near-tie count is recorded."""
    near = {}
    heads = range(g.heads) if heads is None else heads
    members = oracle.tile_members(g)
    for h in heads:
        qm = oracle.tile_means(q[:, h], g, members)
        km = oracle.tile_means(k[:, h], g, members)
        r = np.arange(g.n_tiles) if rows is None else np.asarray(rows)
        sel, gap = oracle.select_tiles(qm, km, keep, rows=r)
        nt = gap < oracle.NEAR_TIE_REL_GAP
        near[h] = r[nt]
        record_near_ties(what or f"{g} keep={keep} head {h}", len(r), int(nt.sum()))
        gs = gpu_sel[h][r]
        assert (gs.sum(1) == keep).all(), "GPU keeps a different number of tiles"
        bad = np.nonzero((gs != sel).any(1) & ~nt)[0]
        assert len(bad) == 0, f"head {h}: {len(bad)} rows differ outside near-ties (first row {r[bad[0]]})"
        # near-tie rows: every kept tile scores >= every dropped tile, up to the gap
        s = qm[r] @ km.T
        for i in np.nonzero(nt)[0]:
            kept = s[i][gs[i]]
            dropped = s[i][~gs[i]]
            if len(dropped):
                lo, hi = kept.min(), dropped.max()
                assert lo >= hi - 1e-5 * max(abs(lo), abs(hi)) - 1e-30
    return near

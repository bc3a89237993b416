"""Seeded synthetic inputs for the Zebra3D global-attention workloads.

This module is shared by the CPU oracle and the CUDA path. It holds only the
input recipes: random draws, the token layout needed to place the synthetic
latent structure, and rounding of the draws to bfloat16-representable values.
It performs none of the attention method's arithmetic.

Workloads (all five follow the configuration texts quoted with the method's
headline metric; the page "How Hybrid Attention Lets Feed-Forward 3D Models
Scale to Many Views" supplies the token structure: per view, special tokens
then an 8x8-tiled patch grid, section "Linear-centered stages plus tile-sparse
stages"):

  tiny_fp32        4 views, 16x16 grid, 2 heads, fp32, seed 0; Q/K/V ~ N(0,1)
                   plus a per-(view-tile, head) offset 2*N(0,1)^d shared by
                   Q, K and V; affine A = I + 0.01*N(0,1), b ~ N(0, 0.01^2).
  sparse_v32       32 views, 32x32 grid, 16 heads, bf16, seed 1; latent
                   L[view//4, tile position, head] ~ N(0,1)^d shared by Q/K/V
                   plus N(0, 0.5^2) token noise; special tokens N(0,1).
  linear_v128      128 views, 37x37 grid, 16 heads, bf16, seed 2; N(0,1);
                   affine drawn as for tiny_fp32.
  sidebyside_v512  512 views, 37x37 grid, 16 heads, bf16, seed 3; latent
                   structure of sparse_v32.
  stack_v1024      1,024 views, 37x37 grid, model dim 1024, 16 heads, bf16,
                   seed 4; x0 ~ N(0,1); per layer W_qkv, W_o ~ N(0, 0.02^2);
                   24 layers; linear layers draw an affine as tiny_fp32.

Large tensors are drawn in fixed token blocks, each from its own PCG64 stream
keyed by (seed, tensor id, block index), so a draw does not depend on the
number of threads used and any block can be regenerated alone.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os

import numpy as np

N_SPECIAL = 5          # 1 camera + 4 register tokens per view
TILE = 8               # 8x8-patch tiles
HEAD_DIM = 64
BLOCK_TOKENS = 32768   # token block of one random stream

# tensor ids of the random streams
_ID_Q, _ID_K, _ID_V, _ID_OFFSET, _ID_LATENT, _ID_A, _ID_B, _ID_X = range(8)
_ID_WQKV, _ID_WO = 100, 200


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    views: int
    grid_h: int
    grid_w: int
    heads: int
    dtype: str            # "f32" or "bf16"
    seed: int
    recipe: str           # "offset", "latent", "iid", "stack"
    y: tuple = ()         # sparsity settings exercised on this workload
    layers: int = 0
    model_dim: int = 0
    n_linear: int = 0     # first n_linear layers run the linear stage

    @property
    def tokens_per_view(self) -> int:
        return N_SPECIAL + self.grid_h * self.grid_w

    @property
    def n_tokens(self) -> int:
        return self.views * self.tokens_per_view


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 4, 16, 16, 2, "f32", 0, "offset", y=(0.6, 0.875, 0.0)),
    "sparse_v32": Workload("sparse_v32", 32, 32, 32, 16, "bf16", 1, "latent", y=(0.8, 0.0)),
    "linear_v128": Workload("linear_v128", 128, 37, 37, 16, "bf16", 2, "iid"),
    "sidebyside_v512": Workload("sidebyside_v512", 512, 37, 37, 16, "bf16", 3, "latent", y=(0.6, 0.8)),
    "stack_v1024": Workload("stack_v1024", 1024, 37, 37, 16, "bf16", 4, "stack", y=(0.8,),
                            layers=24, model_dim=1024, n_linear=17),
}


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns a new float32 array.

    uint32 arithmetic, exact for every finite input (the rounding increment
    cannot carry past the exponent of a finite float); large arrays are
    processed in threaded chunks.
    """
    out = np.array(x, dtype=np.float32, copy=True, order="C")
    u = out.reshape(-1).view(np.uint32)
    step = 1 << 24

    def work(lo):
        seg = u[lo:lo + step]
        inc = (seg >> 16) & 1
        inc += 0x7FFF
        seg += inc
        seg &= 0xFFFF0000

    starts = range(0, u.size, step)
    if u.size > step:
        with _cf.ThreadPoolExecutor(min(_threads(), len(starts))) as ex:
            list(ex.map(work, starts))
    else:
        for lo in starts:
            work(lo)
    return out


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _threads() -> int:
    try:
        return max(1, min(32, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def normal_blocks(shape_tail: tuple, n_rows: int, seed: int, tensor_id: int,
                  scale: float = 1.0, rows=None) -> np.ndarray:
    """N(0, scale^2) float32 array [n_rows, *shape_tail], drawn block by block.

    `rows` (optional, sorted int array) returns only those rows, drawing only
    the blocks that hold them.
    """
    tail = int(np.prod(shape_tail)) if shape_tail else 1
    if rows is not None:
        rows = np.asarray(rows, dtype=np.int64)
        out = np.empty((len(rows), tail), np.float32)
        for b in np.unique(rows // BLOCK_TOKENS):
            lo = b * BLOCK_TOKENS
            hi = min(n_rows, lo + BLOCK_TOKENS)
            blk = _rng(seed, tensor_id, int(b)).standard_normal((hi - lo, tail), np.float32)
            sel = (rows >= lo) & (rows < hi)
            out[sel] = blk[rows[sel] - lo]
        out *= np.float32(scale)
        return out.reshape((len(rows),) + tuple(shape_tail))
    out = np.empty((n_rows, tail), np.float32)
    n_blocks = (n_rows + BLOCK_TOKENS - 1) // BLOCK_TOKENS

    def fill(b):
        lo = b * BLOCK_TOKENS
        hi = min(n_rows, lo + BLOCK_TOKENS)
        _rng(seed, tensor_id, b).standard_normal((hi - lo, tail), np.float32, out=out[lo:hi])
        if scale != 1.0:
            out[lo:hi] *= np.float32(scale)

    if n_blocks <= 1:
        for b in range(n_blocks):
            fill(b)
    else:
        with _cf.ThreadPoolExecutor(min(_threads(), n_blocks)) as ex:
            list(ex.map(fill, range(n_blocks)))
    return out.reshape((n_rows,) + tuple(shape_tail))


def token_tile_position(views: int, grid_h: int, grid_w: int):
    """Per token: (view, tile position within the view or -1 for special tokens).

    Token order inside a view: the special tokens first, then patches in
    row-major grid order; tile position = (row // 8) * ceil(grid_w / 8) + col // 8.
    """
    L = N_SPECIAL + grid_h * grid_w
    j = np.arange(L)
    p = j - N_SPECIAL
    r, c = p // grid_w, p % grid_w
    tc = (grid_w + TILE - 1) // TILE
    pos = np.where(j < N_SPECIAL, -1, (r // TILE) * tc + (c // TILE))
    view = np.repeat(np.arange(views), L)
    return view, np.tile(pos, views)


def qkv(w: Workload, rows=None):
    """Q, K, V as float32 arrays [N, H, 64] (bf16-representable for bf16 workloads).

    `rows` restricts the output to those token indices (same values as in the
    full draw).
    """
    if w.recipe == "stack":
        raise ValueError("the stack workload draws x0 and weights, see stack_inputs()")
    N, H, d = w.n_tokens, w.heads, HEAD_DIM
    sel = np.arange(N) if rows is None else np.asarray(rows, np.int64)
    view, pos = token_tile_position(w.views, w.grid_h, w.grid_w)
    view, pos = view[sel], pos[sel]
    if w.recipe == "iid":
        outs = [normal_blocks((H, d), N, w.seed, t, rows=rows) for t in (_ID_Q, _ID_K, _ID_V)]
    elif w.recipe == "offset":
        tv = ((w.grid_h + TILE - 1) // TILE) * ((w.grid_w + TILE - 1) // TILE)
        off = 2.0 * _rng(w.seed, _ID_OFFSET).standard_normal((w.views * tv, H, d)).astype(np.float32)
        outs = []
        for t in (_ID_Q, _ID_K, _ID_V):
            x = normal_blocks((H, d), N, w.seed, t, rows=rows)
            patch = pos >= 0
            x[patch] += off[view[patch] * tv + pos[patch]]
            outs.append(x)
    elif w.recipe == "latent":
        tv = ((w.grid_h + TILE - 1) // TILE) * ((w.grid_w + TILE - 1) // TILE)
        groups = (w.views + 3) // 4
        lat = _rng(w.seed, _ID_LATENT).standard_normal((groups * tv, H, d)).astype(np.float32)
        outs = []
        for t in (_ID_Q, _ID_K, _ID_V):
            x = normal_blocks((H, d), N, w.seed, t, rows=rows)
            patch = pos >= 0
            x[patch] *= np.float32(0.5)
            x[patch] += lat[(view[patch] // 4) * tv + pos[patch]]
            outs.append(x)
    else:
        raise ValueError(w.recipe)
    if w.dtype == "bf16":
        outs = [round_to_bf16(x) for x in outs]
    return tuple(outs)


def affine(heads: int, seed: int, layer: int = 0, dtype: str = "f32"):
    """Per-head affine correction: A = I + 0.01*N(0,1) [H,64,64], b ~ N(0, 0.01^2) [H,64] (float32)."""
    d = HEAD_DIM
    A = np.eye(d, dtype=np.float32)[None] + np.float32(0.01) * _rng(seed, _ID_A, layer).standard_normal(
        (heads, d, d)).astype(np.float32)
    b = np.float32(0.01) * _rng(seed, _ID_B, layer).standard_normal((heads, d)).astype(np.float32)
    return A.astype(np.float32), b.astype(np.float32)


def stack_x0(w: Workload, rows=None) -> np.ndarray:
    """x0 ~ N(0,1) [N, model_dim] rounded to bf16 (float32 array)."""
    return round_to_bf16(normal_blocks((w.model_dim,), w.n_tokens, w.seed, _ID_X, rows=rows))


def stack_layer_weights(w: Workload, layer: int):
    """(W_qkv [3D, D], W_o [D, D]) ~ N(0, 0.02^2), bf16-rounded float32, for one layer."""
    D = w.model_dim
    wqkv = _rng(w.seed, _ID_WQKV, layer).standard_normal((3 * D, D), np.float32) * np.float32(0.02)
    wo = _rng(w.seed, _ID_WO, layer).standard_normal((D, D), np.float32) * np.float32(0.02)
    return round_to_bf16(wqkv), round_to_bf16(wo)


def stack_layer_kinds(w: Workload):
    """'linear' for the first n_linear layers, 'sparse' for the rest."""
    return ["linear" if i < w.n_linear else "sparse" for i in range(w.layers)]


def custom(views, grid_h, grid_w, heads, seed, recipe="iid", dtype="bf16", name="custom") -> Workload:
    """A workload with another geometry and one of the recipes above."""
    return Workload(name, views, grid_h, grid_w, heads, dtype, seed, recipe)

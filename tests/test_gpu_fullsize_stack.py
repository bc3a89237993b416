"""GPU parity of one stacked tile-sparse layer at the headline size.

The layer is the one the benchmark's seven sparse layers run: 1,024 views of
37x37 patches plus 5 special tokens (N = 1,406,976), model dim 1024, 16 heads,
y = 0.8 (5,120 of 25,600 key tiles kept), QKV projection -> Q/K RMS norm +
2D rotation (fused into the tile packing) -> selection -> tile-sparse attention
and dense special-token rows -> output projection + residual, all through
zebra_hybrid_layer.

Inputs: x = x0 / 16 with x0 the benchmark's seeded N(0,1) input, and the
benchmark's own W_qkv of its first sparse layer (layer 17, N(0, 0.02^2)). W_o
is block-diagonal (one random 64x64 block per head) and large, so that each
head's attention output reaches its own 64 output columns and the attention
term carries >= 90% of the output norm (asserted on the oracle). The oracle
then needs the projections of the sampled heads only: it computes them in
float64 for every token, rounds them to bf16 as the kernel stores them (the tile
selection is a discrete decision, taken in the kernel's precision on both sides),
normalises and rotates them in float64, runs its sparse stage on
8 query tiles (one of each tile shape among them) and 4 special-token rows, and
adds x plus the block of W_o. Selections of the sampled tiles must be
bit-exact outside near-ties.
"""
import numpy as np
import pytest
import torch

import linear_global_attention_b200 as zb
import oracle
import synth
from oracle import Geom
from tests import parity_helpers as ph

pytestmark = pytest.mark.gpu

STACK = synth.WORKLOADS["stack_v1024"]
G = Geom(STACK.views, STACK.grid_h, STACK.grid_w, STACK.heads)
LAYER = STACK.n_linear                     # the first sparse layer of the 0.7L/0.8S stack
Y = STACK.y[0]
HEADS = [0, 9, 15]
WO_SCALE = 128.0                          # std of the W_o blocks


def tiles_sample():
    tv = 25                                # 5 x 5 tiles per 37 x 37 view
    # full (8x8), 8x5, 5x8 and 5x5 tiles in different views, plus four random tiles
    fixed = [3 * tv + 6, 200 * tv + 4, 511 * tv + 20, 1023 * tv + 24]
    rng = np.random.default_rng(1717)
    extra = rng.choice(G.n_tiles, 4, replace=False)
    return np.unique(np.concatenate([fixed, extra]))


def inputs():
    x = synth.stack_x0(STACK) * np.float32(0.0625)         # exact: a power of two
    wqkv, _ = synth.stack_layer_weights(STACK, LAYER)
    rng = np.random.default_rng(1718)
    D = STACK.model_dim
    wo = np.zeros((D, D), np.float32)
    for h in range(STACK.heads):
        wo[h * 64:(h + 1) * 64, h * 64:(h + 1) * 64] = WO_SCALE * rng.standard_normal((64, 64))
    return x, wqkv, synth.round_to_bf16(wo)


def oracle_side(x, wqkv, wo, tiles, specials):
    """x_out at the sampled rows and heads (the heads' 64 output columns each),
    with the oracle's selections and score gaps."""
    D = STACK.model_dim
    cols = np.concatenate([np.arange(s * D + h * 64, s * D + h * 64 + 64) for s in range(3) for h in HEADS])
    w = np.asarray(wqkv[cols], np.float64)
    N, nh = x.shape[0], len(HEADS)
    proj = np.empty((N, len(cols)))
    step = 65536
    for lo in range(0, N, step):
        # the kernel stores the projection in bf16 and selects tiles from those values:
        # the oracle takes the selection in the same precision (arithmetic after it is float64)
        proj[lo:lo + step] = synth.round_to_bf16((np.asarray(x[lo:lo + step], np.float64) @ w.T).astype(np.float32))
    q, k, v = (proj[:, s * nh * 64:(s + 1) * nh * 64].reshape(N, nh, 64) for s in range(3))
    del proj
    gh = Geom(G.views, G.grid_h, G.grid_w, nh)
    qn = oracle.rope_2d(oracle.rms_norm(q), gh)
    kn = oracle.rope_2d(oracle.rms_norm(k), gh)
    keep = oracle.keep_count(Y, G.n_tiles)
    rows, o, sel, gaps = oracle.sparse_stage(qn, kn, v, gh, keep, query_tiles=tiles, special_rows=specials)
    out = np.empty((len(rows), nh, 64))
    for a, h in enumerate(HEADS):
        blk = np.asarray(wo[h * 64:(h + 1) * 64, h * 64:(h + 1) * 64], np.float64)
        out[:, a] = np.asarray(x[rows, h * 64:(h + 1) * 64], np.float64) + o[:, a] @ blk.T
    return rows, out, sel, gaps, keep


def test_stacked_sparse_layer_full_size_sampled():
    x, wqkv, wo = inputs()
    tiles = tiles_sample()
    specials = np.sort(np.random.default_rng(1719).choice(oracle.special_tokens(G), 4, replace=False))
    zg = ph.zgeom(G)
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    out = torch.empty_like(xd)
    ws = zb.workspace(zg, zb.ZEBRA_OP_HYBRID_SPARSE, zb.ZEBRA_BF16, Y)
    zb.zebra_hybrid_layer(zg, zb.ZEBRA_LAYER_SPARSE, xd, torch.from_numpy(wqkv).to(torch.bfloat16).cuda(),
                          torch.from_numpy(wo).to(torch.bfloat16).cuda(), None, None, Y, out, ws)
    torch.cuda.synchronize()
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    del ws, xd
    rows, want, sel, gaps, keep = oracle_side(x, wqkv, wo, tiles, specials)
    assert keep == 5120
    got_all = out[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    tid = oracle.tile_of_token(G)
    for a, h in enumerate(HEADS):
        xr = x[rows, h * 64:(h + 1) * 64].astype(np.float64)
        got = got_all[:, h * 64:(h + 1) * 64]
        share = np.linalg.norm(want[:, a] - xr) / np.linalg.norm(want[:, a])
        assert share >= 0.9, f"head {h}: attention share {share:.3f}"
        near_tiles = tiles[gaps[a] < oracle.NEAR_TIE_REL_GAP]
        ph.record_near_ties(f"full-size stacked sparse head {h}", len(tiles), len(near_tiles))
        ok = ~np.isin(tid[rows], near_tiles)
        ph.assert_close(got[ok], want[ok, a], "bf16", f"full-size stacked sparse head {h}")

"""GPU parity of the attention-concentration diagnostic (zebra_coverage) with
oracle.coverage.

Page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to Many Views",
section "Sensitive stages also concentrate their attention". The GPU selects
key tiles (zebra_tile_pool + zebra_tile_select) and then measures, for every
row of the sampled query tiles, the dense softmax mass on the selected tiles'
tokens and on the special keys. Masses lie in [0, 1]; bf16 Q/K with fp32
accumulation and exponentials give absolute errors far below 1e-4. Tiles whose
oracle selection has a near-tie are counted and left out.
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
ATOL = 1e-4


def _gpu_coverage(g, q, k, y, tiles):
    zg = ph.zgeom(g)
    sel, _, keep, mask = ph.run_select(g, q, k, y, "bf16")
    qd, kd = ph.dev(q, "bf16"), ph.dev(k, "bf16")
    n = len(tiles)
    s_mass = torch.full((n, g.heads, 64), float("nan"), device="cuda")
    p_mass = torch.full_like(s_mass, float("nan"))
    ws = torch.empty(zb.zebra_coverage_workspace_bytes(zg, n), dtype=torch.uint8, device="cuda")
    zb.zebra_coverage(zg, qd, kd, mask, tiles, s_mass, p_mass, ws)
    torch.cuda.synchronize()
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    return sel, keep, s_mass.cpu().numpy().astype(np.float64), p_mass.cpu().numpy().astype(np.float64)


def _compare(g, q, k, y, tiles, heads, label):
    sel, keep, s_mass, p_mass = _gpu_coverage(g, q, k, y, tiles)
    near = ph.check_selection(g, q, k, keep, sel, heads=heads, rows=tiles, what=f"coverage {label}")
    rows, want_sel, want_spec = oracle.coverage(q, k, g, keep, query_tiles=tiles, heads=heads)
    _, _, counts = oracle.tile_members(g)
    got_sel = np.concatenate([s_mass[i, :, :counts[t]].T for i, t in enumerate(tiles)])   # [R, H]
    got_spec = np.concatenate([p_mass[i, :, :counts[t]].T for i, t in enumerate(tiles)])
    row_tile = oracle.tile_of_token(g)[rows]
    for a, h in enumerate(heads):
        ok = ~np.isin(row_tile, near[h])
        np.testing.assert_allclose(got_sel[ok, h], want_sel[ok, a], atol=ATOL, rtol=0)
        np.testing.assert_allclose(got_spec[ok, h], want_spec[ok, a], atol=ATOL, rtol=0)
    # rows beyond a partial tile are zero
    for i, t in enumerate(tiles):
        assert (s_mass[i, :, counts[t]:] == 0).all() and (p_mass[i, :, counts[t]:] == 0).all()
    return got_sel, got_spec


@pytest.mark.parametrize("y", [0.6, 0.9])
def test_coverage_ragged_all_tiles(y):
    g = Geom(6, 21, 19, 4)
    w = synth.custom(6, 21, 19, 4, seed=101, recipe="latent")
    q, k, _ = synth.qkv(w)
    _compare(g, q, k, y, np.arange(g.n_tiles), list(range(g.heads)), f"ragged y={y}")


def test_coverage_y0_covers_everything():
    # every tile kept: the selected and special masses add up to 1 for every row
    g = Geom(4, 16, 16, 2)
    rng = np.random.default_rng(41)
    q, k = (synth.round_to_bf16(rng.standard_normal((g.n_tokens, 2, 64)).astype(np.float32)) for _ in range(2))
    got_sel, got_spec = _compare(g, q, k, 0.0, np.arange(g.n_tiles), [0, 1], "y=0")
    np.testing.assert_allclose(got_sel + got_spec, 1.0, atol=ATOL)


def test_coverage_sparse_v32_sampled():
    w = synth.WORKLOADS["sparse_v32"]
    g = Geom(w.views, w.grid_h, w.grid_w, w.heads)
    q, k, _ = synth.qkv(w)
    tiles = np.sort(np.random.default_rng(42).choice(g.n_tiles, 8, replace=False))
    got_sel, _ = _compare(g, q, k, 0.8, tiles, [0, 7, 15], "v32 y=0.8")
    # the latent recipe concentrates attention: the kept 20% of tiles hold most of the mass
    assert np.median(got_sel) > 0.5

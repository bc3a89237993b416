"""Pins of the oracle's attention-concentration diagnostic (coverage).

Page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to Many Views",
section "Sensitive stages also concentrate their attention": stages are
profiled by how concentrated their attention mass is, and sparse selection
covers most of the relevant mass where it is concentrated. The page defines no
formula and prints no values, so each pin is a closed form or a brute force.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import Geom

G = Geom(3, 11, 13, 2)   # ragged: partial edge tiles


def _qk(seed, g=G):
    r = np.random.default_rng(seed)
    return (r.standard_normal((g.n_tokens, g.heads, 64)) for _ in range(2))


def test_all_tiles_kept_covers_all_patch_mass():
    q, k = _qk(1)
    _, sel, spec = oracle.coverage(q, k, G, G.n_tiles)
    np.testing.assert_allclose(sel + spec, 1.0, atol=1e-12)
    assert (spec > 0).all()


def test_constant_keys_give_the_kept_token_fraction():
    # equal logits: p is uniform over all N keys, so the covered mass is the
    # kept tiles' token count over N
    q, _ = _qk(2)
    k = np.ones_like(q)
    keep = 4
    rows, sel, spec = oracle.coverage(q, k, G, keep)
    order, starts, counts = oracle.tile_members(G)
    tid = oracle.tile_of_token(G)
    for h in range(G.heads):
        qm = oracle.tile_means(q[:, h], G)
        km = oracle.tile_means(k[:, h], G)
        kept, _ = oracle.select_tiles(qm, km, keep)
        want = np.array([counts[kept[tid[i]]].sum() for i in rows]) / G.n_tokens
        np.testing.assert_allclose(sel[:, h], want, atol=1e-12)
        np.testing.assert_allclose(spec[:, h], G.views * G.n_special / G.n_tokens, atol=1e-12)


def test_brute_force_rows():
    # explicit per-key loop with the 1/sqrt(d) scale for a few rows
    q, k = _qk(3)
    keep = 5
    tiles = [0, 6, 11]
    rows, sel, spec = oracle.coverage(q, k, G, keep, query_tiles=tiles, heads=[1])
    tid = oracle.tile_of_token(G)
    qm = oracle.tile_means(q[:, 1], G)
    km = oracle.tile_means(k[:, 1], G)
    kept, _ = oracle.select_tiles(qm, km, keep, rows=np.array(tiles))
    for r in (0, len(rows) // 2, len(rows) - 1):
        i = rows[r]
        logits = [sum(q[i, 1, c] * k[j, 1, c] for c in range(64)) / math.sqrt(64) for j in range(G.n_tokens)]
        mx = max(logits)
        w = [math.exp(x - mx) for x in logits]
        z = sum(w)
        row_kept = kept[tiles.index(int(tid[i]))]
        want_sel = sum(w[j] for j in range(G.n_tokens) if tid[j] >= 0 and row_kept[tid[j]]) / z
        want_spec = sum(w[j] for j in range(G.n_tokens) if tid[j] < 0) / z
        assert abs(sel[r, 0] - want_sel) < 1e-12
        assert abs(spec[r, 0] - want_spec) < 1e-12


def test_concentrated_queries_are_covered():
    # queries of tile 0 point at the keys of tile 5, which then wins the
    # selection and holds almost all of the mass
    q, k = _qk(4)
    order, starts, counts = oracle.tile_members(G)
    direction = np.random.default_rng(5).standard_normal(64)
    direction /= np.linalg.norm(direction)
    for i in order[starts[0]:starts[0] + counts[0]]:
        q[i, 0] = 8.0 * direction
    for j in order[starts[5]:starts[5] + counts[5]]:
        k[j, 0] = 8.0 * direction
    _, sel, _ = oracle.coverage(q, k, G, 1, query_tiles=[0], heads=[0])
    assert sel.min() > 0.99


@pytest.mark.parametrize("seed", [6, 7])
def test_coverage_grows_with_the_kept_fraction(seed):
    # the kept sets are nested (top-k of the same scores), so covered mass
    # never shrinks as more tiles are kept
    q, k = _qk(seed)
    prev = None
    for keep in (1, 3, 8, G.n_tiles):
        _, sel, _ = oracle.coverage(q, k, G, keep)
        if prev is not None:
            assert (sel >= prev - 1e-12).all()
        prev = sel

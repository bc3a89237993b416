"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test ties one part of the oracle to something independent: the
workloads' stated token/tile counts, a textbook or library routine that the
method reduces to in a special case, a closed form, an exhaustive search, or
a pure-Python brute force written here from the method's description.
Method source: page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to
Many Views", sections "Linear-centered stages plus tile-sparse stages" (tiles,
selector, landmarks, visibility rules), "A closed-form fit avoids retraining
from scratch" (affine correction) and "Speedup scales with the number of
input views" (Q/K normalisation, positional rotation, channel-softmax phi).
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import Geom

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand_qkv(g: Geom, seed: int, scale=1.0):
    rng = np.random.default_rng(seed)
    shp = (g.n_tokens, g.heads, g.head_dim)
    return tuple(scale * rng.standard_normal(shp) for _ in range(3))


# ---------------------------------------------------------------------------
# Geometry: stated counts
# ---------------------------------------------------------------------------
def _golden_geometry():
    rows = []
    with open(os.path.join(HERE, "golden", "geometry.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, V, gh, gw, N, tv, full, shapes = line.split()
            rows.append((name, int(V), int(gh), int(gw), int(N), int(tv), int(full), shapes))
    return rows


@pytest.mark.parametrize("row", _golden_geometry(), ids=lambda r: r[0])
def test_geometry_matches_stated_counts(row):
    name, V, gh, gw, N, tv, full, shapes = row
    w = synth.WORKLOADS[name]
    assert (w.views, w.grid_h, w.grid_w) == (V, gh, gw)
    g = Geom(V, gh, gw, 2)
    assert g.n_tokens == N == w.n_tokens
    assert g.tiles_per_view == tv
    _, _, counts = oracle.tile_members(g)
    per_view = counts[:tv]
    assert (per_view == 64).sum() == full
    # tile shapes from the partition itself: rows x cols per tile of view 0
    special, view, r, c = oracle.token_coords(g)
    tid = oracle.tile_of_token(g)
    got = {}
    for u in range(tv):
        m = tid == u
        key = f"{len(np.unique(r[m]))}x{len(np.unique(c[m]))}"
        got[key] = got.get(key, 0) + 1
    want = dict(s.split(":") for s in shapes.split(","))
    assert got == {k: int(v) for k, v in want.items()}
    assert counts.sum() == V * gh * gw


def test_tile_index_is_row_major_and_views_do_not_mix():
    g = Geom(3, 11, 19, 1)
    tid = oracle.tile_of_token(g)
    special, view, r, c = oracle.token_coords(g)
    # brute force: walk the grid of each view
    u = 0
    for vw in range(3):
        for br in range(0, 11, 8):
            for bc in range(0, 19, 8):
                toks = [vw * g.tokens_per_view + 5 + rr * 19 + cc
                        for rr in range(br, min(br + 8, 11)) for cc in range(bc, min(bc + 8, 19))]
                assert set(np.nonzero(tid == u)[0]) == set(toks)
                u += 1
    assert u == g.n_tiles
    assert (tid[special] == -1).all() and special.sum() == 3 * 5


# ---------------------------------------------------------------------------
# Selector
# ---------------------------------------------------------------------------
def test_keep_count_rule():
    assert oracle.keep_count(0.6, 16) == 7          # ceil(0.4 * 16) = ceil(6.4)
    assert oracle.keep_count(0.875, 16) == 2
    assert oracle.keep_count(0.0, 16) == 16
    assert oracle.keep_count(0.8, 512) == 103       # ceil(102.4)
    assert oracle.keep_count(0.8, 25600) == 5120
    assert oracle.keep_count(0.6, 12800) == 5120
    assert oracle.keep_count(0.8, 12800) == 2560
    assert oracle.keep_count(0.9999, 4) == 1
    with pytest.raises(ValueError):
        oracle.keep_count(1.0, 4)


@pytest.mark.parametrize("seed", range(6))
def test_selector_against_exhaustive_subset_search(seed):
    rng = np.random.default_rng(seed)
    T = 7
    d = 3
    # integer-valued means make exact score ties common
    qm = rng.integers(-2, 3, size=(T, d)).astype(float)
    km = rng.integers(-2, 3, size=(T, d)).astype(float)
    s = qm @ km.T
    for keep in range(1, T + 1):
        sel, _ = oracle.select_tiles(qm, km, keep)
        for t in range(T):
            best = None
            for subset in itertools.combinations(range(T), keep):   # lexicographic order
                tot = sum(s[t, u] for u in subset)
                if best is None or tot > best[0]:
                    best = (tot, subset)
            assert set(np.nonzero(sel[t])[0]) == set(best[1]), (keep, t)


def test_selector_near_tie_gap():
    qm = np.array([[1.0, 0.0]])
    km = np.array([[1.0, 0.0], [1.0 - 1e-7, 0.0], [0.5, 0.0]])
    sel, gap = oracle.select_tiles(qm, km, 1)
    assert sel[0].tolist() == [True, False, False]
    assert gap[0] == pytest.approx(1e-7, rel=1e-6)
    _, gap2 = oracle.select_tiles(qm, km, 2)
    assert gap2[0] == pytest.approx((0.5 - 1e-7) / (1 - 1e-7), rel=1e-9)


def test_tile_means_against_direct_loops():
    g = Geom(2, 10, 13, 1)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((g.n_tokens, 64))
    m = oracle.tile_means(x, g)
    u = 0
    for vw in range(2):
        for br in range(0, 10, 8):
            for bc in range(0, 13, 8):
                toks = [vw * g.tokens_per_view + 5 + rr * 13 + cc
                        for rr in range(br, min(br + 8, 10)) for cc in range(bc, min(bc + 8, 13))]
                np.testing.assert_allclose(m[u], x[toks].mean(0), rtol=0, atol=1e-14)
                u += 1


# ---------------------------------------------------------------------------
# Sparse stage
# ---------------------------------------------------------------------------
def _sdpa_dense(q, k, v):
    """Dense softmax attention by torch's library routine, in float64 on the CPU."""
    qt = torch.from_numpy(np.ascontiguousarray(q.transpose(1, 0, 2)))[None]
    kt = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2)))[None]
    vt = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2)))[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    return o[0].numpy().transpose(1, 0, 2)


@pytest.mark.parametrize("geom", [Geom(4, 16, 16, 2), Geom(3, 13, 11, 2), Geom(2, 3, 2, 1)],
                         ids=["tiny", "ragged", "subtile"])
def test_y0_equals_dense_softmax_attention(geom):
    q, k, v = _rand_qkv(geom, 5, scale=1.5)
    out = oracle.sparse_stage_full(q, k, v, geom, geom.n_tiles)
    np.testing.assert_allclose(out, _sdpa_dense(q, k, v), rtol=0, atol=1e-12)


def test_y0_equals_dense_on_tiny_workload():
    w = synth.WORKLOADS["tiny_fp32"]
    g = Geom(w.views, w.grid_h, w.grid_w, w.heads)
    q, k, v = (x.astype(np.float64) for x in synth.qkv(w))
    out = oracle.sparse_stage_full(q, k, v, g, oracle.keep_count(0.0, g.n_tiles))
    np.testing.assert_allclose(out, _sdpa_dense(q, k, v), rtol=0, atol=1e-12)


@pytest.mark.parametrize("keep", [1, 3, 9])
def test_constant_keys_give_the_global_value_mean(keep):
    """All keys equal: exact logits are equal and landmark logits add ln(m), so the
    softmax weights are proportional to the number of tokens each entry stands for.
    If every token is represented exactly once, every output row is the mean of all
    N values (closed form)."""
    g = Geom(3, 12, 9, 2)
    rng = np.random.default_rng(11)
    q = rng.standard_normal((g.n_tokens, 2, 64))
    k = np.broadcast_to(rng.standard_normal((1, 2, 64)), q.shape).copy()
    v = rng.standard_normal(q.shape)
    qm = rng.standard_normal((g.n_tiles, 64))  # irrelevant: selection is forced below
    out_rows, out, _, _ = oracle.sparse_stage(q, k, v, g, keep)
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(0), out.shape), rtol=0, atol=1e-12)
    # also with a random forced selection that leaves some own tiles unselected
    forced = {h: rng.random((g.n_tiles, g.n_tiles)) < 0.3 for h in range(2)}
    for h in range(2):
        np.fill_diagonal(forced[h], False)
    _, out2, _, _ = oracle.sparse_stage(q, k, v, g, keep, force_selected=forced)
    np.testing.assert_allclose(out2, np.broadcast_to(v.mean(0), out2.shape), rtol=0, atol=1e-12)
    del qm


def test_constant_tiles_selected_equals_summarised():
    """Every tile holds identical K/V rows: a landmark then equals its tile's tokens
    exactly, so any selection gives dense attention."""
    g = Geom(2, 11, 14, 2)
    rng = np.random.default_rng(7)
    tid = oracle.tile_of_token(g)
    q = rng.standard_normal((g.n_tokens, 2, 64))
    kt = rng.standard_normal((g.n_tiles, 2, 64))
    vt = rng.standard_normal((g.n_tiles, 2, 64))
    k = rng.standard_normal(q.shape)
    v = rng.standard_normal(q.shape)
    patch = tid >= 0
    k[patch] = kt[tid[patch]]
    v[patch] = vt[tid[patch]]
    dense = _sdpa_dense(q, k, v)
    for trial in range(3):
        forced = {h: rng.random((g.n_tiles, g.n_tiles)) < 0.4 for h in range(2)}
        _, out, _, _ = oracle.sparse_stage(q, k, v, g, 1, force_selected=forced)
        np.testing.assert_allclose(out, dense, rtol=0, atol=1e-12)


def _brute_force_sparse(q, k, v, g: Geom, keep: int):
    """Pure-Python per-query construction of the visible set, written from the
    method's description independently of the oracle's vectorised code."""
    N, H, d = q.shape
    L = g.n_special + g.grid_h * g.grid_w
    tc = (g.grid_w + 7) // 8
    tr = (g.grid_h + 7) // 8
    tv = tr * tc

    def tile(n):
        j = n % L
        if j < g.n_special:
            return None
        p = j - g.n_special
        return (n // L) * tv + (p // g.grid_w // 8) * tc + (p % g.grid_w) // 8

    tiles = {}
    for n in range(N):
        u = tile(n)
        if u is not None:
            tiles.setdefault(u, []).append(n)
    T = len(tiles)
    specials = [n for n in range(N) if tile(n) is None]
    out = np.zeros((N, H, d))
    for h in range(H):
        mean = lambda x, toks: sum(x[n, h] for n in toks) / len(toks)  # noqa: E731
        qm = [mean(q, tiles[u]) for u in range(T)]
        km = [mean(k, tiles[u]) for u in range(T)]
        for n in range(N):
            entries = []   # (logit, value)
            t = tile(n)
            if t is None:
                for m in range(N):
                    entries.append((float(q[n, h] @ k[m, h]) / 8.0, v[m, h]))
            else:
                scores = [(-float(qm[t] @ km[u]), u) for u in range(T)]
                chosen = {u for _, u in sorted(scores)[:keep]}
                for u in range(T):
                    if u in chosen:
                        for m in tiles[u]:
                            entries.append((float(q[n, h] @ k[m, h]) / 8.0, v[m, h]))
                    else:
                        rest = [m for m in tiles[u] if m != n]
                        if u == t:
                            entries.append((float(q[n, h] @ k[n, h]) / 8.0, v[n, h]))
                        if rest:
                            kk = sum(k[m, h] for m in rest) / len(rest)
                            vv = sum(v[m, h] for m in rest) / len(rest)
                            entries.append((float(q[n, h] @ kk) / 8.0 + math.log(len(rest)), vv))
                for m in specials:
                    entries.append((float(q[n, h] @ k[m, h]) / 8.0, v[m, h]))
            mx = max(e[0] for e in entries)
            w = [math.exp(e[0] - mx) for e in entries]
            out[n, h] = sum(wi * e[1] for wi, e in zip(w, entries)) / sum(w)
    return out


@pytest.mark.parametrize("geom,keep", [(Geom(2, 9, 10, 1), 2), (Geom(2, 9, 10, 2), 5),
                                       (Geom(3, 1, 1, 1), 1), (Geom(1, 17, 3, 1), 2)],
                         ids=["ragged-k2", "ragged-k5", "one-token-tiles", "narrow"])
def test_sparse_stage_against_brute_force(geom, keep):
    q, k, v = _rand_qkv(geom, 21, scale=1.3)
    # make some own tiles lose the selection: shift key means away from query means
    out = oracle.sparse_stage_full(q, k, v, geom, keep)
    ref = _brute_force_sparse(q, k, v, geom, keep)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # the own-tile-unselected branch must have been exercised
    sel = oracle.select_tiles(oracle.tile_means(q[:, 0], geom), oracle.tile_means(k[:, 0], geom), keep)[0]
    if keep < geom.n_tiles:
        assert (~np.diag(sel)).any()


def test_sampled_rows_equal_full_run():
    g = Geom(3, 12, 12, 2)
    q, k, v = _rand_qkv(g, 2)
    full = oracle.sparse_stage_full(q, k, v, g, 4)
    rows, out, _, _ = oracle.sparse_stage(q, k, v, g, 4, query_tiles=[1, 5], special_rows=[0, 151])
    np.testing.assert_allclose(out, full[rows], rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# Linear stage pieces
# ---------------------------------------------------------------------------
def test_phi_is_a_channel_softmax():
    from scipy.special import softmax
    x = np.random.default_rng(0).standard_normal((50, 64)) * 4
    p = oracle.phi(x)
    assert (p > 0).all()
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(p, softmax(x, axis=-1), rtol=1e-13, atol=0)
    np.testing.assert_allclose(oracle.phi(x + 3.0), p, rtol=1e-12)


def test_rms_norm_unit_rms_and_scale_invariance():
    x = np.random.default_rng(1).standard_normal((40, 64)) * 3
    y = oracle.rms_norm(x, 0.0)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(-1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(oracle.rms_norm(5 * x, 0.0), y, rtol=1e-13)
    # eps enters under the root: for mean(x^2) = 1e-6 the output RMS is 1/sqrt(2)
    z = np.full((1, 64), 1e-3)
    np.testing.assert_allclose(np.sqrt((oracle.rms_norm(z, 1e-6) ** 2).mean()), 1 / math.sqrt(2), rtol=1e-12)


def test_rope_matches_complex_rotation_and_base_100():
    g = Geom(2, 6, 7, 1)
    rng = np.random.default_rng(4)
    x = rng.standard_normal((g.n_tokens, 64))
    y = oracle.rope_2d(x, g, 100.0)
    special, _, r, c = oracle.token_coords(g)
    j = np.arange(16)
    theta = np.array([100.0 ** (-jj / 16.0) for jj in j])   # 100^(-2j/32)
    for n in range(g.n_tokens):
        if special[n]:
            np.testing.assert_array_equal(y[n], x[n])
            continue
        for off, pos in ((0, r[n]), (32, c[n])):
            z = x[n, off:off + 16] + 1j * x[n, off + 16:off + 32]
            w = z * np.exp(1j * pos * theta)
            np.testing.assert_allclose(y[n, off:off + 16], w.real, atol=1e-13)
            np.testing.assert_allclose(y[n, off + 16:off + 32], w.imag, atol=1e-13)
    # pair 0 turns by exactly 1 rad per row step; pair 8 by 100^(-1/2) = 0.1 rad
    e = np.zeros((g.n_tokens, 64))
    e[:, 0] = 1.0
    e[:, 8] = 1.0
    ye = oracle.rope_2d(e, g, 100.0)
    n = 5 + 1 * 7 + 0          # view 0, row 1, col 0
    assert ye[n, 0] == pytest.approx(math.cos(1.0)) and ye[n, 16] == pytest.approx(math.sin(1.0))
    assert ye[n, 8] == pytest.approx(math.cos(0.1)) and ye[n, 24] == pytest.approx(math.sin(0.1))


def test_rope_norm_preserving_and_relative():
    g = Geom(1, 9, 9, 1)
    rng = np.random.default_rng(8)
    a = rng.standard_normal(64)
    b = rng.standard_normal(64)
    xa = np.broadcast_to(a, (g.n_tokens, 64))
    xb = np.broadcast_to(b, (g.n_tokens, 64))
    ra = oracle.rope_2d(xa, g)
    rb = oracle.rope_2d(xb, g)
    np.testing.assert_allclose(np.linalg.norm(ra, axis=1), np.linalg.norm(a), rtol=1e-13)
    _, _, r, c = oracle.token_coords(g)
    tok = lambda rr, cc: 5 + rr * 9 + cc  # noqa: E731
    assert np.allclose(ra[tok(0, 0)], a)
    # <R(p) a, R(p') b> depends only on p - p'
    base = ra[tok(3, 5)] @ rb[tok(1, 2)]
    assert base == pytest.approx(ra[tok(5, 8)] @ rb[tok(3, 5)], rel=1e-12)
    assert base == pytest.approx(ra[tok(2, 3)] @ rb[tok(0, 0)], rel=1e-12)


def test_linear_stage_equals_explicit_kernel_product():
    """Associativity check: phi(Q) (phi(K)^T V) / phi(Q) sum phi(K) equals the
    explicit N x N normalised kernel matrix applied to V, then the affine map."""
    g = Geom(2, 6, 5, 2)
    q, k, v = _rand_qkv(g, 9)
    A, b = synth.affine(2, 9)
    out = oracle.linear_stage(q, k, v, g, A, b)
    for h in range(2):
        fq = oracle.linear_features(q[:, h], g)
        fk = oracle.linear_features(k[:, h], g)
        W = fq @ fk.T                       # [N, N]
        W = W / W.sum(1, keepdims=True)
        o = W @ v[:, h]
        np.testing.assert_allclose(out[:, h], o @ A[h].astype(np.float64).T + b[h], rtol=0, atol=1e-12)


def test_linear_stage_constant_features_closed_form():
    """A 1x1 grid has no rotation; with identical keys every phi(k) is equal, so the
    linear stage returns A mean(V) + b for every query."""
    g = Geom(5, 1, 1, 1)
    rng = np.random.default_rng(12)
    q = rng.standard_normal((g.n_tokens, 1, 64))
    k = np.broadcast_to(rng.standard_normal((1, 1, 64)), q.shape)
    v = rng.standard_normal(q.shape)
    A, b = synth.affine(1, 12)
    out = oracle.linear_stage(q, k, v, g, A, b)
    want = A[0].astype(np.float64) @ v[:, 0].mean(0) + b[0]
    np.testing.assert_allclose(out[:, 0], np.broadcast_to(want, out[:, 0].shape), atol=1e-12)


def test_linear_stage_sampled_rows():
    g = Geom(2, 9, 9, 2)
    q, k, v = _rand_qkv(g, 14)
    A, b = synth.affine(2, 14)
    full = oracle.linear_stage(q, k, v, g, A, b)
    rows = np.array([0, 3, 7, 60, 171])
    np.testing.assert_allclose(oracle.linear_stage(q, k, v, g, A, b, rows=rows), full[rows], rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# Stacked hybrid layer
# ---------------------------------------------------------------------------
def _layer_inputs(g: Geom, seed: int):
    rng = np.random.default_rng(seed)
    D = g.heads * 64
    x = rng.standard_normal((g.n_tokens, D))
    wqkv = 0.05 * rng.standard_normal((3 * D, D))
    wo = 0.05 * rng.standard_normal((D, D))
    return x, wqkv, wo


def test_hybrid_dense_layer_against_library_composition():
    g = Geom(2, 8, 9, 2)
    x, wqkv, wo = _layer_inputs(g, 1)
    out = oracle.hybrid_layer(x, wqkv, wo, "dense", g)
    qkv = torch.from_numpy(x) @ torch.from_numpy(wqkv).T
    D = 128
    q, k, v = (qkv[:, i * D:(i + 1) * D].reshape(-1, 2, 64) for i in range(3))
    rms = lambda t: t * torch.rsqrt((t * t).mean(-1, keepdim=True) + 1e-6)  # noqa: E731
    qn = torch.from_numpy(oracle.rope_2d(rms(q).numpy(), g))
    kn = torch.from_numpy(oracle.rope_2d(rms(k).numpy(), g))
    o = torch.nn.functional.scaled_dot_product_attention(qn.transpose(0, 1)[None], kn.transpose(0, 1)[None],
                                                         v.transpose(0, 1)[None])[0].transpose(0, 1)
    want = torch.from_numpy(x) + o.reshape(-1, D) @ torch.from_numpy(wo).T
    np.testing.assert_allclose(out, want.numpy(), rtol=0, atol=1e-11)


def test_hybrid_sparse_y0_equals_dense_and_zero_wo_is_identity():
    g = Geom(2, 8, 9, 2)
    x, wqkv, wo = _layer_inputs(g, 2)
    d = oracle.hybrid_layer(x, wqkv, wo, "dense", g)
    s = oracle.hybrid_layer(x, wqkv, wo, "sparse", g, keep=g.n_tiles)
    np.testing.assert_allclose(s, d, rtol=0, atol=1e-11)
    A, b = synth.affine(2, 2)
    for kind in ("dense", "sparse", "linear"):
        out = oracle.hybrid_layer(x, wqkv, np.zeros_like(wo), kind, g, A=A, b=b, keep=3)
        np.testing.assert_array_equal(out, x)


def test_hybrid_linear_layer_uses_linear_stage_on_projections():
    g = Geom(2, 5, 6, 2)
    x, wqkv, wo = _layer_inputs(g, 3)
    A, b = synth.affine(2, 3)
    out = oracle.hybrid_layer(x, wqkv, wo, "linear", g, A=A, b=b)
    # composition by the library: torch matmuls around the plain kernel-product form
    qkv = x @ wqkv.T
    q, k, v = (qkv[:, i * 128:(i + 1) * 128].reshape(-1, 2, 64) for i in range(3))
    o = np.zeros_like(q)
    for h in range(2):
        fq = oracle.linear_features(q[:, h], g)
        fk = oracle.linear_features(k[:, h], g)
        W = fq @ fk.T
        o[:, h] = (W / W.sum(1, keepdims=True)) @ v[:, h] @ A[h].astype(np.float64).T + b[h]
    want = (torch.from_numpy(x) + torch.from_numpy(o.reshape(-1, 128)) @ torch.from_numpy(wo).T).numpy()
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-11)

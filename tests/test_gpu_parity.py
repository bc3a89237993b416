"""GPU parity of every C-ABI entry point against the fp64 oracle, on seeded
synthetic inputs small enough for the oracle to finish in seconds yet spanning
several tiles, partial edge tiles and the degenerate cases of the method."""
import numpy as np
import pytest
import torch

import linear_global_attention_b200 as zb
import oracle
import synth
from oracle import Geom
from tests import hybrid_cases as hc
from tests import parity_helpers as ph

pytestmark = pytest.mark.gpu


def _w(name):
    w = synth.WORKLOADS[name]
    return w, Geom(w.views, w.grid_h, w.grid_w, w.heads)


RAGGED = synth.custom(6, 21, 19, 4, seed=101, recipe="latent", name="ragged")
RAGGED_G = Geom(6, 21, 19, 4)


@pytest.fixture(scope="module")
def ragged_inputs():
    return synth.qkv(RAGGED)


@pytest.fixture(scope="module")
def tiny_inputs():
    return synth.qkv(synth.WORKLOADS["tiny_fp32"])


# ---------------------------------------------------------------------------
# pooling / packing
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_tile_pool_means_and_packing(ragged_inputs, dtype):
    g = RAGGED_G
    q = ragged_inputs[0]
    zg = ph.zgeom(g)
    T = g.n_tiles
    x = ph.dev(q, dtype)
    mean = torch.empty(g.heads, T, 64, device="cuda")
    packed = torch.full((g.heads, T, 64, 64), 7.0, dtype=x.dtype, device="cuda")
    counts = torch.empty(T, dtype=torch.int32, device="cuda")
    zb.zebra_tile_pool(zg, x, mean, packed, counts)
    torch.cuda.synchronize()
    order, starts, cnt = oracle.tile_members(g)
    assert (counts.cpu().numpy() == cnt).all()
    # packing moves values only: exact
    want = np.zeros((g.heads, T, 64, 64), np.float32)
    for u in range(T):
        toks = order[starts[u]:starts[u] + cnt[u]]
        want[:, u, :cnt[u]] = q[toks].transpose(1, 0, 2)
    np.testing.assert_array_equal(packed.float().cpu().numpy(), want)
    for h in range(g.heads):
        m = oracle.tile_means(q[:, h], g)
        np.testing.assert_allclose(mean[h].cpu().numpy(), m, rtol=0, atol=2e-6)


def test_tile_pool_strided_input(ragged_inputs):
    """A [N, 3, H, d] buffer viewed per tensor, like the split of a QKV projection."""
    g = RAGGED_G
    q, k, v = ragged_inputs
    big = ph.dev(np.stack([q, k, v], axis=1).reshape(g.n_tokens, 3 * g.heads, 64), "bf16")
    kview = big[:, g.heads:2 * g.heads, :]
    mean = torch.empty(g.heads, g.n_tiles, 64, device="cuda")
    zb.zebra_tile_pool(ph.zgeom(g), kview, mean)
    torch.cuda.synchronize()
    for h in range(g.heads):
        np.testing.assert_allclose(mean[h].cpu().numpy(), oracle.tile_means(k[:, h], g), rtol=0, atol=2e-6)


# ---------------------------------------------------------------------------
# selector
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("y", [0.0, 0.6, 0.875, 0.99])
def test_select_bit_exact_ragged(ragged_inputs, y):
    q, k, _ = ragged_inputs
    sel, nt, keep, _ = ph.run_select(RAGGED_G, q, k, y, "bf16")
    assert keep == oracle.keep_count(y, RAGGED_G.n_tiles)
    ph.check_selection(RAGGED_G, q, k, keep, sel)


def test_select_ties_go_to_the_lower_index():
    g = Geom(5, 12, 12, 2)
    rng = np.random.default_rng(0)
    q = rng.standard_normal((g.n_tokens, 2, 64)).astype(np.float32)
    k = np.ones_like(q)            # every key tile has the same mean: all scores tie
    sel, nt, keep, _ = ph.run_select(g, q, k, 0.6, "f32")
    assert keep == 8
    want = np.zeros(g.n_tiles, bool)
    want[:keep] = True
    assert (sel == want).all()
    assert nt.all()                # a full tie is a near-tie


@pytest.mark.parametrize("tied", [3000, 700, 100], ids=["crowded_bin", "sorted_ties", "ranked_ties"])
def test_select_threshold_ties(tied):
    """Key means built so that `tied` key tiles score exactly the same for every
    query tile and the keep-th score falls inside that group: the group lands in
    one histogram bin (more than 1,024 keys: the radix passes; up to 1,024: the
    exact sort of the bin; up to 256: the one-pass ranks), and equal scores must
    go to the lower tile index on both sides. The other key tiles score far from
    the tied value, so the comparison is exact for every row."""
    g = Geom(60, 64, 64, 1)                       # 3,840 tiles (only the geometry matters here)
    T = g.n_tiles
    rng = np.random.default_rng(61)
    q_mean = np.abs(rng.standard_normal((1, T, 64))).astype(np.float32) + 0.5
    base = np.full(64, 0.25, np.float32)
    k_mean = np.empty((1, T, 64), np.float32)
    order = rng.permutation(T)
    tied_idx, rest = order[:tied], order[tied:]
    k_mean[0, tied_idx] = base                      # identical key means: identical scores
    hi = rest[: (T - tied) // 2]
    lo = rest[(T - tied) // 2:]
    k_mean[0, hi] = base + 1.0 + rng.random((len(hi), 64)).astype(np.float32)   # clearly above
    k_mean[0, lo] = base - 1.0 - rng.random((len(lo), 64)).astype(np.float32)   # clearly below
    keep = len(hi) + tied // 3                      # the cut falls inside the tied group
    y = 1.0 - (keep - 0.5) / T
    assert oracle.keep_count(y, T) == keep
    zg = ph.zgeom(g)
    qd, kd = torch.from_numpy(q_mean).cuda(), torch.from_numpy(k_mean).cuda()
    mask = torch.empty((1, T, zg.mask_words), dtype=torch.int32, device="cuda")
    ws = zb.workspace(zg, zb.ZEBRA_OP_SELECT, zb.ZEBRA_BF16, y)
    got_keep = zb.zebra_tile_select(zg, qd, kd, y, mask, None, ws)
    torch.cuda.synchronize()
    assert got_keep == keep
    gsel = ph.unpack_mask(mask, T)[0]
    want, _ = oracle.select_tiles(q_mean[0].astype(np.float64), k_mean[0].astype(np.float64), keep)
    assert (gsel == want).all()
    # the tie rule: exactly the lowest-index members of the tied group are kept
    first = np.sort(tied_idx)[: keep - len(hi)]
    assert gsel[:, first].all() and not gsel[:, np.setdiff1d(tied_idx, first)].any()


def test_select_sparse_v32_full():
    w, g = _w("sparse_v32")
    q, k, _ = synth.qkv(w)
    sel, nt, keep, _ = ph.run_select(g, q, k, 0.8, "bf16")
    assert keep == 103
    near = ph.check_selection(g, q, k, keep, sel)
    n_near = sum(len(v) for v in near.values())
    assert n_near <= 0.05 * g.heads * g.n_tiles


# ---------------------------------------------------------------------------
# sparse stage
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("y", [0.6, 0.875, 0.0])
def test_sparse_tiny_fp32(tiny_inputs, y):
    w, g = _w("tiny_fp32")
    q, k, v = tiny_inputs
    out = ph.host(ph.run_sparse(g, q, k, v, y, "f32"))
    keep = oracle.keep_count(y, g.n_tiles)
    want = oracle.sparse_stage_full(q, k, v, g, keep)
    ph.assert_close(out, want, "f32", f"tiny fp32 y={y}")


@pytest.mark.parametrize("y", [0.6, 0.875, 0.0])
def test_sparse_tiny_bf16(tiny_inputs, y):
    w, g = _w("tiny_fp32")
    q, k, v = (synth.round_to_bf16(x) for x in tiny_inputs)
    out = ph.host(ph.run_sparse(g, q, k, v, y, "bf16"))
    want = oracle.sparse_stage_full(q, k, v, g, oracle.keep_count(y, g.n_tiles))
    ph.assert_close(out, want, "bf16", f"tiny bf16 y={y}")


@pytest.mark.parametrize("y", [0.6, 0.9])
def test_sparse_ragged_bf16(ragged_inputs, y):
    g = RAGGED_G
    q, k, v = ragged_inputs
    keep = oracle.keep_count(y, g.n_tiles)
    out = ph.host(ph.run_sparse(g, q, k, v, y, "bf16"))
    sel, _, _, _ = ph.run_select(g, q, k, y, "bf16")
    near = ph.check_selection(g, q, k, keep, sel)
    want = oracle.sparse_stage_full(q, k, v, g, keep)
    tid = oracle.tile_of_token(g)
    for h in range(g.heads):
        ok = ~np.isin(tid, near[h])
        ph.assert_close(out[ok, h], want[ok, h], "bf16", f"ragged y={y} head {h}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_sparse_own_tile_unselected_branch(dtype):
    """iid inputs at high sparsity: many query tiles do not keep their own tile, so
    the exact self key and the own-tile landmark of the other n_t - 1 tokens are used."""
    g = Geom(5, 19, 21, 3)
    w = synth.custom(5, 19, 21, 3, seed=55, recipe="iid", dtype="bf16" if dtype == "bf16" else "f32")
    q, k, v = synth.qkv(w)
    y = 0.9
    keep = oracle.keep_count(y, g.n_tiles)
    own = np.stack([oracle.select_tiles(oracle.tile_means(q[:, h], g), oracle.tile_means(k[:, h], g),
                                        keep)[0].diagonal() for h in range(g.heads)])
    assert (~own).sum() >= g.n_tiles      # the branch is exercised many times
    out = ph.host(ph.run_sparse(g, q, k, v, y, dtype))
    sel, _, _, _ = ph.run_select(g, q, k, y, dtype)
    near = ph.check_selection(g, q, k, keep, sel)
    want = oracle.sparse_stage_full(q, k, v, g, keep)
    tid = oracle.tile_of_token(g)
    for h in range(g.heads):
        ok = ~np.isin(tid, near[h])
        ph.assert_close(out[ok, h], want[ok, h], dtype, f"own-tile branch head {h}")


def test_sparse_fp32_ragged_matches_tightly(ragged_inputs):
    g = RAGGED_G
    q, k, v = ragged_inputs
    out = ph.host(ph.run_sparse(g, q, k, v, 0.7, "f32"))
    keep = oracle.keep_count(0.7, g.n_tiles)
    sel, _, _, _ = ph.run_select(g, q, k, 0.7, "f32")
    near = ph.check_selection(g, q, k, keep, sel)
    want = oracle.sparse_stage_full(q, k, v, g, keep)
    tid = oracle.tile_of_token(g)
    for h in range(g.heads):
        ok = ~np.isin(tid, near[h])
        ph.assert_close(out[ok, h], want[ok, h], "f32", f"fp32 ragged head {h}")


def test_sparse_caller_mask_is_used(ragged_inputs):
    g = RAGGED_G
    q, k, v = ragged_inputs
    _, _, _, mask = ph.run_select(g, q, k, 0.75, "bf16")
    a = ph.run_sparse(g, q, k, v, 0.75, "bf16")
    b = ph.run_sparse(g, q, k, v, 0.75, "bf16", mask=mask)
    assert torch.equal(a, b)


def test_sparse_v32_sampled():
    w, g = _w("sparse_v32")
    q, k, v = synth.qkv(w)
    keep = oracle.keep_count(0.8, g.n_tiles)
    out = ph.host(ph.run_sparse(g, q, k, v, 0.8, "bf16"))
    rng = np.random.default_rng(7)
    tiles = np.sort(rng.choice(g.n_tiles, 12, replace=False))
    specials = np.sort(rng.choice(oracle.special_tokens(g), 8, replace=False))
    heads = [0, 5, 15]
    rows, want, sel, gaps = oracle.sparse_stage(q, k, v, g, keep, query_tiles=tiles, special_rows=specials,
                                                heads=heads)
    tid = oracle.tile_of_token(g)
    for h in heads:
        near_tiles = tiles[gaps[h] < oracle.NEAR_TIE_REL_GAP]
        ph.record_near_ties(f"v32 sampled head {h}", len(tiles), len(near_tiles))
        ok = ~np.isin(tid[rows], near_tiles)
        ph.assert_close(out[rows][ok, h], want[ok, h], "bf16", f"v32 head {h}")


def test_sparse_y0_equals_dense_sdpa():
    w, g = _w("sparse_v32")
    q, k, v = synth.qkv(w)
    out = ph.run_sparse(g, q, k, v, 0.0, "bf16").float()
    qt, kt, vt = (ph.dev(x, "f32").transpose(0, 1)[None] for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0].transpose(0, 1)
    ph.assert_close(out.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64), "bf16",
                    "y=0 vs SDPA")


# ---------------------------------------------------------------------------
# degenerate geometries
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("geom,y", [
    (Geom(5, 1, 1, 2), 0.5),          # one-token tiles: own-tile landmark empty
    (Geom(3, 3, 5, 2), 0.5),          # one partial tile per view
    (Geom(4, 9, 17, 2, n_special=0), 0.7),   # no special tokens
    (Geom(2, 40, 33, 1), 0.99),       # keep a single tile
    (Geom(1, 8, 8, 3), 0.0),          # one view, one tile
    (Geom(7, 13, 6, 2, n_special=1), 0.3),
], ids=["1x1", "3x5", "nospecial", "keep1", "single", "odd"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_sparse_degenerate(geom, y, dtype):
    rng = np.random.default_rng(3)
    shp = (geom.n_tokens, geom.heads, 64)
    q, k, v = (rng.standard_normal(shp).astype(np.float32) for _ in range(3))
    if dtype == "bf16":
        q, k, v = (synth.round_to_bf16(x) for x in (q, k, v))
    keep = oracle.keep_count(y, geom.n_tiles)
    out = ph.host(ph.run_sparse(geom, q, k, v, y, dtype))
    sel, _, _, _ = ph.run_select(geom, q, k, y, dtype)
    near = ph.check_selection(geom, q, k, keep, sel)
    want = oracle.sparse_stage_full(q, k, v, geom, keep)
    tid = oracle.tile_of_token(geom)
    for h in range(geom.heads):
        ok = ~np.isin(tid, near[h])
        ph.assert_close(out[ok, h], want[ok, h], dtype, f"{geom} head {h}")


def test_sparse_constant_tiles_invariant():
    """Tiles with identical K/V rows: any selection gives dense attention."""
    g = Geom(4, 12, 10, 2)
    rng = np.random.default_rng(5)
    tid = oracle.tile_of_token(g)
    q = rng.standard_normal((g.n_tokens, 2, 64)).astype(np.float32)
    k = rng.standard_normal(q.shape).astype(np.float32)
    v = rng.standard_normal(q.shape).astype(np.float32)
    kt = rng.standard_normal((g.n_tiles, 2, 64)).astype(np.float32)
    vt = rng.standard_normal((g.n_tiles, 2, 64)).astype(np.float32)
    p = tid >= 0
    k[p], v[p] = kt[tid[p]], vt[tid[p]]
    dense = ph.host(ph.run_sparse(g, q, k, v, 0.0, "f32"))
    for y in (0.5, 0.9):
        out = ph.host(ph.run_sparse(g, q, k, v, y, "f32"))
        ph.assert_close(out, dense, "f32", f"constant tiles y={y}")


def test_sparse_is_deterministic(ragged_inputs):
    g = RAGGED_G
    q, k, v = ragged_inputs
    a = ph.run_sparse(g, q, k, v, 0.6, "bf16")
    b = ph.run_sparse(g, q, k, v, 0.6, "bf16")
    assert torch.equal(a, b)


def test_empty_views_is_a_noop():
    g = zb.geom(0, 16, 16, 2)
    x = torch.empty(0, 2, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    zb.zebra_sparse_attn(g, x, x, x, 0.5, x, ws)
    zb.zebra_linear_attn(g, x, x, x, None, None, x, ws)


# ---------------------------------------------------------------------------
# linear stage
# ---------------------------------------------------------------------------
def _run_linear(g, q, k, v, A, b, dtype):
    zg = ph.zgeom(g)
    qd, kd, vd = ph.dev(q, dtype), ph.dev(k, dtype), ph.dev(v, dtype)
    out = torch.empty_like(qd)
    ws = zb.workspace(zg, zb.ZEBRA_OP_LINEAR, zb.ZEBRA_BF16 if dtype == "bf16" else zb.ZEBRA_F32)
    At = None if A is None else torch.from_numpy(A).cuda()
    bt = None if b is None else torch.from_numpy(b).cuda()
    zb.zebra_linear_attn(zg, qd, kd, vd, At, bt, out, ws)
    torch.cuda.synchronize()
    return ph.host(out)


def test_linear_tiny_fp32(tiny_inputs):
    w, g = _w("tiny_fp32")
    q, k, v = tiny_inputs
    A, b = synth.affine(g.heads, w.seed)
    out = _run_linear(g, q, k, v, A, b, "f32")
    ph.assert_close(out, oracle.linear_stage(q, k, v, g, A, b), "f32", "linear tiny fp32")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_linear_ragged(ragged_inputs, dtype):
    g = RAGGED_G
    q, k, v = ragged_inputs
    A, b = synth.affine(g.heads, 101)
    out = _run_linear(g, q, k, v, A, b, dtype)
    ph.assert_close(out, oracle.linear_stage(q, k, v, g, A, b), dtype, f"linear ragged {dtype}")


def test_linear_identity_affine_defaults(ragged_inputs):
    g = RAGGED_G
    q, k, v = ragged_inputs
    out = _run_linear(g, q, k, v, None, None, "bf16")
    eye = np.broadcast_to(np.eye(64, dtype=np.float32), (g.heads, 64, 64)).copy()
    ph.assert_close(out, oracle.linear_stage(q, k, v, g, eye, np.zeros((g.heads, 64), np.float32)), "bf16",
                    "linear identity")


def test_linear_v128_full_size_sampled():
    w, g = _w("linear_v128")
    q, k, v = synth.qkv(w)
    A, b = synth.affine(g.heads, w.seed)
    out = _run_linear(g, q, k, v, A, b, "bf16")
    rng = np.random.default_rng(2)
    rows = np.sort(rng.choice(g.n_tokens, 4000, replace=False))
    heads = [0, 7, 15]
    want = oracle.linear_stage(q, k, v, g, A, b, rows=rows, heads=heads)
    for h in heads:
        ph.assert_close(out[rows, h], want[:, h], "bf16", f"linear v128 head {h}")


def test_linear_head_stride_zero_copy_path():
    """Heads aliased by a head stride of 0: no tensor map describes that layout, so the state kernel
    loads K and V by its 16-byte asynchronous copies instead of bulk tensor copies."""
    g = Geom(4, 21, 19, 3)
    rng = np.random.default_rng(17)
    one = [synth.round_to_bf16(rng.standard_normal((g.n_tokens, 1, 64)).astype(np.float32)) for _ in range(3)]
    q, k, v = (np.ascontiguousarray(np.broadcast_to(x, (g.n_tokens, g.heads, 64))) for x in one)
    A, b = synth.affine(g.heads, 17)
    zg = ph.zgeom(g)
    qd, kd, vd = (torch.from_numpy(x).to(torch.bfloat16).cuda().expand(g.n_tokens, g.heads, 64) for x in one)
    assert qd.stride(1) == 0
    out = torch.empty((g.n_tokens, g.heads, 64), dtype=torch.bfloat16, device="cuda")
    ws = zb.workspace(zg, zb.ZEBRA_OP_LINEAR, zb.ZEBRA_BF16)
    zb.zebra_linear_attn(zg, qd, kd, vd, torch.from_numpy(A).cuda(), torch.from_numpy(b).cuda(), out, ws)
    torch.cuda.synchronize()
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    ph.assert_close(ph.host(out), oracle.linear_stage(q, k, v, g, A, b), "bf16", "linear, head stride 0")


@pytest.mark.parametrize("geom", [Geom(3, 1, 1, 2), Geom(2, 3, 5, 1, n_special=0), Geom(1, 40, 33, 2)],
                         ids=["1x1", "nospecial", "wide"])
def test_linear_degenerate(geom):
    rng = np.random.default_rng(9)
    shp = (geom.n_tokens, geom.heads, 64)
    q, k, v = (synth.round_to_bf16(rng.standard_normal(shp).astype(np.float32)) for _ in range(3))
    A, b = synth.affine(geom.heads, 9)
    out = _run_linear(geom, q, k, v, A, b, "bf16")
    ph.assert_close(out, oracle.linear_stage(q, k, v, geom, A, b), "bf16", f"linear {geom}")


# ---------------------------------------------------------------------------
# stacked hybrid layer
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("kind", ["linear", "sparse", "dense"])
def test_hybrid_layer_small(kind):
    """One stacked layer of each kind against the oracle, on inputs where the
    attention term carries >= 90% of the output norm (tests/hybrid_cases.py),
    so the Q/K normalisation, the rotation and the attention itself are visible
    at the bf16 tolerance (tests/test_hybrid_sensitivity.py plants those
    mistakes in the oracle and checks that they fail this comparison)."""
    g = hc.GEOM
    x, wqkv, wo, A, b = hc.small_case()
    _, want = hc.oracle_out(kind)
    assert hc.attention_share(x, want) >= hc.MIN_ATTN_SHARE
    zg = ph.zgeom(g)
    kinds = {"linear": zb.ZEBRA_LAYER_LINEAR, "sparse": zb.ZEBRA_LAYER_SPARSE, "dense": zb.ZEBRA_LAYER_DENSE}
    ops = {"linear": zb.ZEBRA_OP_HYBRID_LINEAR, "sparse": zb.ZEBRA_OP_HYBRID_SPARSE, "dense": zb.ZEBRA_OP_HYBRID_DENSE}
    xd = ph.dev(x, "bf16")
    out = torch.empty_like(xd)
    ws = zb.workspace(zg, ops[kind], zb.ZEBRA_BF16, hc.Y)
    zb.zebra_hybrid_layer(zg, kinds[kind], xd, ph.dev(wqkv, "bf16"), ph.dev(wo, "bf16"),
                          torch.from_numpy(A).cuda(), torch.from_numpy(b).cuda(), hc.Y, out, ws)
    torch.cuda.synchronize()
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    got = ph.host(out)
    ph.assert_close(got, want, "bf16", f"hybrid {kind}")
    # the attention term alone (x_out - x) within the same bar, relative to its own norm
    ph.assert_close(got - x, want - x, "bf16", f"hybrid {kind} attention term")


def test_hybrid_in_place():
    g = Geom(3, 9, 9, 2)
    D = 128
    rng = np.random.default_rng(4)
    x = synth.round_to_bf16(rng.standard_normal((g.n_tokens, D)).astype(np.float32))
    wqkv = synth.round_to_bf16((0.02 * rng.standard_normal((3 * D, D))).astype(np.float32))
    wo = synth.round_to_bf16((0.02 * rng.standard_normal((D, D))).astype(np.float32))
    zg = ph.zgeom(g)
    ws = zb.workspace(zg, zb.ZEBRA_OP_HYBRID_LINEAR)
    xd = ph.dev(x, "bf16")
    out = torch.empty_like(xd)
    W1, W2 = ph.dev(wqkv, "bf16"), ph.dev(wo, "bf16")
    zb.zebra_hybrid_layer(zg, zb.ZEBRA_LAYER_LINEAR, xd, W1, W2, None, None, 0.0, out, ws)
    zb.zebra_hybrid_layer(zg, zb.ZEBRA_LAYER_LINEAR, xd, W1, W2, None, None, 0.0, xd, ws)
    torch.cuda.synchronize()
    assert torch.equal(out, xd)


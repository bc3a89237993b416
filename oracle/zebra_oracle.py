"""Plain fp64 CPU oracle of the Zebra3D multi-view global-attention layer.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
baseline may import this module; the library path never calls it and shares
no code with it. It is deliberately slow and direct: NumPy float64, per-tile
Python loops, no blocking or fusion beyond what the method states.

Source: the page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to
Many Views" (wispaper.ai, English; its Chinese version says the same), cited
below by section title:
  [GA]  "Global attention dominates runtime as views grow"
  [LC]  "Linear-centered stages plus tile-sparse stages"
  [CF]  "A closed-form fit avoids retraining from scratch"
  [SP]  "Speedup scales with the number of input views"
  [SC]  "Sensitive stages also concentrate their attention"
The Chinese page's section on linear and tile-sparse layers adds that each
*complete* tile holds 64 tokens, i.e. edge tiles may be partial.

Readings of points the page leaves open (each marked READING below):
  R1 token order: per view, 5 special tokens (1 camera, 4 register) first,
     then the patch grid in row-major order.
  R2 tiles: 8x8 patch blocks anchored at grid (0, 0); bottom/right edge tiles
     are partial; tiles never cross views; tile index
     u = view * T_v + (row // 8) * ceil(W / 8) + col // 8.
  R3 selection is per (head, query tile) over all T patch tiles of all views,
     own tile included; special tokens are never candidates.
  R4 tile score = unscaled dot of the mean-pooled query and mean-pooled key of
     the tile (means over the tile's actual tokens).
  R5 keep count k = clamp(ceil((1 - y) * T - 1e-6), 1, T).
  R6 equal scores: the lower tile index wins.
  R7 partition rule: every key token is seen exactly once, either exactly or
     inside one landmark; when a query's own tile is not selected, its self
     key is exact and the own-tile landmark covers the other n_t - 1 tokens.
  R8 landmark logit = q . k_mean / sqrt(d) + ln(m), m = tokens it represents;
     a landmark with m = 0 is omitted.
  R9 softmax scale 1/sqrt(d) for exact keys and landmarks alike.
  R10 Q/K normalisation = RMS norm x / sqrt(mean(x^2) + eps), eps = 1e-6, no gain.
  R11 2D rotary positions: channels 0-31 rotate by patch row, 32-63 by patch
     column (0-based within the view); in each 32-channel half the pairs
     (j, j+16), j = 0..15, turn by angle pos * base^(-2j/32); base 100;
     special tokens are not rotated.
  R12 prologue order: normalise, rotate, then phi.
  R13 phi(x)_c = exp(x_c) / sum_c' exp(x_c') (no temperature).
  R14 the linear state sums over all N tokens (special tokens included).
  R15 affine correction applied per head as y = A o + b (o a column vector);
     the centring belongs to the fit.
  R16 in a stacked layer all three kinds (linear, sparse, dense) apply the
     Q/K RMS norm and the rotation before attention.
  R17 stacked layer body: x + W_o Attn(split(W_qkv x)); no bias, no MLP.
  R20 affine fit samples [CF]: one sample per (token, view, scene, head) is
     the pair (x, y) of 64-vectors, x the converted linear output before the
     correction and y the teacher (dense softmax) output; samples of all heads
     are pooled into one fit ("accumulated across ... heads"), and a per-head
     fit is offered as an option.
  R21 centred regularised least squares [CF]: with means mu_x, mu_y and
     covariances C_xx = mean((x-mu_x)(x-mu_x)^T), C_xy = mean((x-mu_x)(y-mu_y)^T)
     over the n accumulated samples, A^T = (C_xx + lam I)^-1 C_xy and
     b = mu_y - A mu_x; lam >= 0 is a parameter (the page gives no value).
  R22 attention concentration [SC]: the coverage of a stage is the dense
     softmax probability mass (scale 1/sqrt(d), all N keys) that a patch query
     puts on the tokens of its query tile's selected key tiles, averaged over
     queries (and heads); the mass on special-token keys is reported apart.
  R23 layer allocation [LC]: the single-stage linear-conversion error of a
     stage is the mean, over its fit samples, of |A x + b - y|^2 (the
     converted output after its fitted correction against the teacher); for a
     requested linear fraction x of L stages, the round(x * L) stages with the
     smallest error (ties: lower stage index) become linear, the rest sparse.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

NEAR_TIE_REL_GAP = 1e-5


# ----------------------------------------------------------------------------
# Geometry: token layout and tile partition  ([LC]; READINGS R1, R2)
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Geom:
    views: int
    grid_h: int
    grid_w: int
    heads: int
    head_dim: int = 64
    n_special: int = 5
    tile: int = 8

    @property
    def patches(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def tokens_per_view(self) -> int:
        return self.n_special + self.patches

    @property
    def n_tokens(self) -> int:
        return self.views * self.tokens_per_view

    @property
    def tile_rows(self) -> int:
        return -(-self.grid_h // self.tile)

    @property
    def tile_cols(self) -> int:
        return -(-self.grid_w // self.tile)

    @property
    def tiles_per_view(self) -> int:
        return self.tile_rows * self.tile_cols

    @property
    def n_tiles(self) -> int:
        return self.views * self.tiles_per_view


def token_coords(g: Geom):
    """Per token: (is_special, view, patch row, patch col); row/col are -1 for special tokens."""
    N, L = g.n_tokens, g.tokens_per_view
    n = np.arange(N)
    view = n // L
    j = n % L
    special = j < g.n_special
    p = j - g.n_special
    row = np.where(special, -1, p // g.grid_w)
    col = np.where(special, -1, p % g.grid_w)
    return special, view, row, col


def tile_of_token(g: Geom) -> np.ndarray:
    """Tile index of every token (R2); -1 for special tokens."""
    special, view, row, col = token_coords(g)
    u = view * g.tiles_per_view + (row // g.tile) * g.tile_cols + (col // g.tile)
    return np.where(special, -1, u)


def tile_members(g: Geom):
    """(order, starts, counts): tokens of tile u are order[starts[u]:starts[u]+counts[u]],
    increasing token index, i.e. row-major inside the tile."""
    tid = tile_of_token(g)
    patch = np.nonzero(tid >= 0)[0]
    order = patch[np.argsort(tid[patch], kind="stable")]
    counts = np.bincount(tid[patch], minlength=g.n_tiles)
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]])
    return order, starts, counts


def special_tokens(g: Geom) -> np.ndarray:
    special, _, _, _ = token_coords(g)
    return np.nonzero(special)[0]


# ----------------------------------------------------------------------------
# Tile pooling  ([LC]: omitted tiles are summarised by their mean key/value)
# ----------------------------------------------------------------------------
def tile_means(x_h: np.ndarray, g: Geom, members=None) -> np.ndarray:
    """Mean over each tile's actual tokens of one head's [N, d] tensor -> [T, d] float64."""
    order, starts, counts = members if members is not None else tile_members(g)
    x = np.asarray(x_h, dtype=np.float64)[order]
    sums = np.add.reduceat(x, starts, axis=0) if len(order) else np.zeros((0, x.shape[1]))
    return sums / counts[:, None]


# ----------------------------------------------------------------------------
# Selector  ([LC]: the selector retains a key-tile fraction of 1 - y; R3-R6)
# ----------------------------------------------------------------------------
def keep_count(y: float, n_tiles: int) -> int:
    """Number of kept key tiles per query tile for sparsity y (READING R5)."""
    if not (0.0 <= y < 1.0):
        raise ValueError("y must lie in [0, 1)")
    k = math.ceil((1.0 - y) * n_tiles - 1e-6)
    return int(min(max(k, 1), n_tiles))


def select_tiles(q_mean: np.ndarray, k_mean: np.ndarray, keep: int, rows=None):
    """Top-`keep` key tiles per query tile by q_mean . k_mean, ties to the lower index.

    Returns (selected [R, T] bool, rel_gap [R]): rel_gap is the relative gap
    between the keep-th and (keep+1)-th scores (inf when keep == T), the
    quantity by which near-ties are recognised.
    """
    q_mean = np.asarray(q_mean, np.float64)
    k_mean = np.asarray(k_mean, np.float64)
    rows = np.arange(q_mean.shape[0]) if rows is None else np.asarray(rows)
    T = k_mean.shape[0]
    s = q_mean[rows] @ k_mean.T                      # [R, T] scores
    order = np.argsort(-s, axis=1, kind="stable")    # descending; equal scores keep index order
    sel = np.zeros(s.shape, bool)
    np.put_along_axis(sel, order[:, :keep], True, axis=1)
    if keep < T:
        a = np.take_along_axis(s, order[:, keep - 1:keep], axis=1)[:, 0]
        b = np.take_along_axis(s, order[:, keep:keep + 1], axis=1)[:, 0]
        den = np.maximum(np.abs(a), np.abs(b))
        gap = np.where(den > 0, np.abs(a - b) / np.where(den > 0, den, 1.0), 0.0)
    else:
        gap = np.full(len(rows), np.inf)
    return sel, gap


# ----------------------------------------------------------------------------
# Softmax helper
# ----------------------------------------------------------------------------
def _softmax_weighted_sum(logits: np.ndarray, values: np.ndarray) -> np.ndarray:
    """Row-wise softmax(logits) @ values, with the row maximum subtracted first."""
    m = logits.max(axis=-1, keepdims=True)
    p = np.exp(logits - m)
    return (p @ values) / p.sum(axis=-1, keepdims=True)


def dense_attention(q_h, k_h, v_h, rows=None) -> np.ndarray:
    """Plain softmax(q k^T / sqrt(d)) v for one head; `rows` selects query rows
    (processed a few at a time so that one block of logits stays near 64 MB)."""
    k_h = np.asarray(k_h, np.float64)
    v_h = np.asarray(v_h, np.float64)
    q_h = np.asarray(q_h, np.float64)
    rows = np.arange(q_h.shape[0]) if rows is None else np.asarray(rows)
    d = q_h.shape[-1]
    chunk = max(1, min(1024, (1 << 23) // max(k_h.shape[0], 1)))
    out = np.empty((len(rows), d))
    for a in range(0, len(rows), chunk):
        r = rows[a:a + chunk]
        out[a:a + chunk] = _softmax_weighted_sum(q_h[r] @ k_h.T / math.sqrt(d), v_h)
    return out


# ----------------------------------------------------------------------------
# Tile-sparse softmax stage  ([LC])
# ----------------------------------------------------------------------------
def sparse_stage(q, k, v, g: Geom, keep: int, query_tiles=None, special_rows=None, heads=None,
                 force_selected=None):
    """Tile-sparse attention of one layer.

    q, k, v: [N, H, d] arrays. Patch queries of the tiles in `query_tiles`
    (default all) attend, per head:
      - every token of the `keep` selected key tiles, exactly;
      - every special-token key, exactly;
      - their own key exactly when their own tile is not selected;
      - one mean-K/V landmark per unselected tile, logit + ln(m) (R7, R8).
    Special-token queries in `special_rows` (default all) attend all N keys
    densely.

    `force_selected` ({h: [Tq, T] bool}, optional) replaces the selector's
    choice, so that tests can vary the selection alone.

    Returns (rows, out, selected, rel_gap): rows = sorted token indices that
    were computed, out [len(rows), H, d] float64, selected {h: [Tq, T] bool}
    and rel_gap {h: [Tq]} for the computed query tiles (in `query_tiles` order).
    """
    N, H, d = q.shape
    assert N == g.n_tokens and H == g.heads and d == g.head_dim
    T = g.n_tiles
    heads = range(H) if heads is None else heads
    query_tiles = np.arange(T) if query_tiles is None else np.asarray(query_tiles)
    specials = special_tokens(g)
    special_rows = specials if special_rows is None else np.asarray(special_rows)
    order, starts, counts = tile_members(g)
    members = (order, starts, counts)
    scale = 1.0 / math.sqrt(d)

    q_rows = np.concatenate([order[starts[t]:starts[t] + counts[t]] for t in query_tiles]) \
        if len(query_tiles) else np.zeros(0, np.int64)
    rows = np.sort(np.concatenate([q_rows, special_rows]).astype(np.int64))
    pos = {int(r): i for i, r in enumerate(rows)}
    out = np.full((len(rows), H, d), np.nan)
    selected, gaps = {}, {}

    for h in heads:
        qh = np.asarray(q[:, h, :], np.float64)
        kh = np.asarray(k[:, h, :], np.float64)
        vh = np.asarray(v[:, h, :], np.float64)
        q_mean = tile_means(qh, g, members)
        k_mean = tile_means(kh, g, members)
        v_mean = tile_means(vh, g, members)
        sel, gap = select_tiles(q_mean, k_mean, keep, rows=query_tiles)
        if force_selected is not None:
            sel = np.asarray(force_selected[h], bool)
        selected[h], gaps[h] = sel, gap
        k_spec, v_spec = kh[specials], vh[specials]

        for a, t in enumerate(query_tiles):
            mine = order[starts[t]:starts[t] + counts[t]]
            Qt = qh[mine]                                              # [n_t, d]
            chosen = np.nonzero(sel[a])[0]
            exact = np.concatenate([order[starts[u]:starts[u] + counts[u]] for u in chosen]
                                   + [np.zeros(0, np.int64)])
            lm = np.array([u for u in range(T) if not sel[a, u] and u != t], dtype=np.int64)
            keys = np.concatenate([kh[exact], k_spec, k_mean[lm]])
            vals = np.concatenate([vh[exact], v_spec, v_mean[lm]])
            bias = np.concatenate([np.zeros(len(exact) + len(specials)), np.log(counts[lm])])
            logits = Qt @ keys.T * scale + bias                         # [n_t, E], shared entries
            ex_logits = np.zeros((len(mine), 0))                        # per-query entries
            ex_values = np.zeros((len(mine), 0, d))
            if not sel[a, t]:
                # own tile unselected: exact self key + landmark of the other n_t - 1 tokens (R7)
                n_t = counts[t]
                self_logit = np.einsum("ij,ij->i", Qt, kh[mine]) * scale
                extra_logits = [self_logit[:, None]]
                extra_values = [vh[mine][:, None, :]]
                if n_t > 1:
                    m = n_t - 1
                    k_rest = (kh[mine].sum(0)[None, :] - kh[mine]) / m
                    v_rest = (vh[mine].sum(0)[None, :] - vh[mine]) / m
                    extra_logits.append((np.einsum("ij,ij->i", Qt, k_rest) * scale + math.log(m))[:, None])
                    extra_values.append(v_rest[:, None, :])
                ex_logits = np.concatenate(extra_logits, axis=1)
                ex_values = np.concatenate(extra_values, axis=1)
            # one softmax over the shared and the per-query entries together
            mx = np.maximum(logits.max(axis=1, initial=-np.inf), ex_logits.max(axis=1, initial=-np.inf))[:, None]
            p = np.exp(logits - mx)
            pe = np.exp(ex_logits - mx)
            num = p @ vals + np.einsum("ie,ied->id", pe, ex_values)
            o = num / (p.sum(axis=1, keepdims=True) + pe.sum(axis=1, keepdims=True))
            for i, n in enumerate(mine):
                out[pos[int(n)], h] = o[i]

        if len(special_rows):
            # special-token query rows keep dense attention over all N keys
            o = dense_attention(qh, kh, vh, rows=special_rows)
            for i, n in enumerate(special_rows):
                out[pos[int(n)], h] = o[i]
    return rows, out, selected, gaps


def sparse_stage_full(q, k, v, g: Geom, keep: int) -> np.ndarray:
    """sparse_stage over every query, as a dense [N, H, d] float64 array."""
    rows, out, _, _ = sparse_stage(q, k, v, g, keep)
    assert len(rows) == g.n_tokens
    return out


# ----------------------------------------------------------------------------
# Linear stage  ([SP]: Q/K normalisation, positional rotation, channel-softmax
# feature map; [GA]/[LC]: linear attention; [CF]: centered affine correction)
# ----------------------------------------------------------------------------
def rms_norm(x, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis (READING R10)."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope_2d(x, g: Geom, base: float = 100.0, rows=None) -> np.ndarray:
    """2D rotary positions on patch tokens of x [R, ..., d] (READING R11).

    x holds the tokens `rows` (default: all N tokens, in order).
    """
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    half, quarter = d // 2, d // 4
    special, _, row, col = token_coords(g)
    if rows is not None:
        special, row, col = special[rows], row[rows], col[rows]
    theta = base ** (-2.0 * np.arange(quarter) / half)               # [16]
    out = x.copy()
    extra = (1,) * (x.ndim - 2)
    for off, pos in ((0, row), (half, col)):
        ang = np.where(special, 0.0, pos)[:, None] * theta[None, :]  # [R, 16]
        c = np.cos(ang).reshape((len(ang),) + extra + (quarter,))
        s = np.sin(ang).reshape((len(ang),) + extra + (quarter,))
        a = x[..., off:off + quarter]
        b = x[..., off + quarter:off + half]
        out[..., off:off + quarter] = a * c - b * s
        out[..., off + quarter:off + half] = b * c + a * s
    return out


def phi(x) -> np.ndarray:
    """Channel softmax feature map over the last axis (READING R13)."""
    x = np.asarray(x, np.float64)
    e = np.exp(x - x.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def linear_features(x, g: Geom, rope_base: float = 100.0, eps: float = 1e-6, rows=None) -> np.ndarray:
    """phi(rope(rms_norm(x))) in the order norm -> rotation -> phi (READING R12)."""
    return phi(rope_2d(rms_norm(x, eps), g, rope_base, rows=rows))


def linear_stage(q, k, v, g: Geom, A, b, rope_base: float = 100.0, eps: float = 1e-6,
                 rows=None, heads=None) -> np.ndarray:
    """Linear global attention with the per-head affine correction.

    Per head: S = sum_n phi(k_n) v_n^T (d x d), z = sum_n phi(k_n) over all N
    tokens (R14); o_n = S^T phi(q_n) / (z . phi(q_n)); y_n = A o_n + b (R15).
    Returns [len(rows), H, d] float64 (rows default: all tokens).
    """
    N, H, d = q.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    heads = range(H) if heads is None else heads
    out = np.full((len(rows), H, d), np.nan)
    for h in heads:
        fk = linear_features(k[:, h, :], g, rope_base, eps)
        fq = linear_features(np.asarray(q[rows, h, :]), g, rope_base, eps, rows=rows)
        vh = np.asarray(v[:, h, :], np.float64)
        S = fk.T @ vh
        z = fk.sum(axis=0)
        o = (fq @ S) / (fq @ z)[:, None]
        out[:, h] = o @ np.asarray(A[h], np.float64).T + np.asarray(b[h], np.float64)
    return out


# ----------------------------------------------------------------------------
# Stacked hybrid layer  ([LC]: xL/yS allocation, preserved projections,
# normalisation and positional encoding; READINGS R16, R17)
# ----------------------------------------------------------------------------
def split_heads(qkv, heads: int, d: int = 64):
    N = qkv.shape[0]
    D = heads * d
    return tuple(qkv[:, i * D:(i + 1) * D].reshape(N, heads, d) for i in range(3))


def hybrid_layer(x, w_qkv, w_o, kind: str, g: Geom, A=None, b=None, keep=None,
                 rope_base: float = 100.0, eps: float = 1e-6, qkv_round=None) -> np.ndarray:
    """x + concat_heads(Attn(split(x W_qkv^T))) W_o^T for one layer of kind
    'linear' | 'sparse' | 'dense'. x [N, D]; w_qkv [3D, D]; w_o [D, D].

    qkv_round (optional) maps the projection output to the precision in which
    an implementation stores it before the attention. The tile selection is a
    discrete decision taken on those stored values, so a comparison with such an
    implementation takes it in the same precision; the arithmetic after it stays
    float64."""
    x = np.asarray(x, np.float64)
    qkv = x @ np.asarray(w_qkv, np.float64).T
    if qkv_round is not None:
        qkv = np.asarray(qkv_round(qkv), np.float64)
    q, k, v = split_heads(qkv, g.heads, g.head_dim)
    N = x.shape[0]
    if kind == "linear":
        o = linear_stage(q, k, v, g, A, b, rope_base, eps)
    else:
        qn = rope_2d(rms_norm(q, eps), g, rope_base)
        kn = rope_2d(rms_norm(k, eps), g, rope_base)
        if kind == "sparse":
            o = sparse_stage_full(qn, kn, v, g, keep)
        elif kind == "dense":
            o = np.stack([dense_attention(qn[:, h], kn[:, h], v[:, h]) for h in range(g.heads)], axis=1)
        else:
            raise ValueError(kind)
    return x + o.reshape(N, -1) @ np.asarray(w_o, np.float64).T


# ----------------------------------------------------------------------------
# closed-form centred affine fit [CF]
# ----------------------------------------------------------------------------
def affine_moments(x, y, per_head: bool = False) -> dict:
    """Accumulable raw moments of the fit samples (READING R20).

    x, y: [n, H, d] (any float type, taken as float64). Returns float64 arrays
    n [G], sx [G, d], sy [G, d], sxx [G, d, d], sxy [G, d, d] with G = H for a
    per-head fit and G = 1 when the heads are pooled. Moments of several calls
    (calibration scenes) add up with affine_moments_add.
    """
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    n, H, d = x.shape
    if per_head:
        xs = [x[:, h] for h in range(H)]
        ys = [y[:, h] for h in range(H)]
    else:
        xs = [x.reshape(n * H, d)]
        ys = [y.reshape(n * H, d)]
    return {
        "n": np.array([float(xi.shape[0]) for xi in xs]),
        "sx": np.stack([xi.sum(0) for xi in xs]),
        "sy": np.stack([yi.sum(0) for yi in ys]),
        "sxx": np.stack([xi.T @ xi for xi in xs]),
        "sxy": np.stack([xi.T @ yi for xi, yi in zip(xs, ys)]),
        "syy": np.array([float((yi * yi).sum()) for yi in ys]),
    }


def affine_moments_add(m1: dict, m2: dict) -> dict:
    """Moments of the union of two sample sets."""
    return {k: m1[k] + m2[k] for k in m1}


def affine_solve(m: dict, lam: float):
    """A [G, d, d] and b [G, d] of the centred ridge fit from raw moments (READING R21)."""
    out_a, out_b = [], []
    for gi in range(m["n"].shape[0]):
        n = m["n"][gi]
        mu_x = m["sx"][gi] / n
        mu_y = m["sy"][gi] / n
        cxx = m["sxx"][gi] / n - np.outer(mu_x, mu_x)
        cxy = m["sxy"][gi] / n - np.outer(mu_x, mu_y)
        a_t = np.linalg.solve(cxx + lam * np.eye(cxx.shape[0]), cxy)
        A = a_t.T
        out_a.append(A)
        out_b.append(mu_y - A @ mu_x)
    return np.stack(out_a), np.stack(out_b)


def affine_fit(x, y, lam: float, per_head: bool = False):
    """Centred affine correction fitted to samples x -> y (READINGS R20, R21)."""
    return affine_solve(affine_moments(x, y, per_head), lam)


# ----------------------------------------------------------------------------
# attention concentration: dense mass covered by the selected tiles [SC]
# ----------------------------------------------------------------------------
def coverage(q, k, g: Geom, keep: int, query_tiles=None, heads=None):
    """Dense softmax mass of patch queries on their selected key tiles (READING R22).

    For every query row of the query tiles `query_tiles` (default: all) and
    head in `heads` (default: all): p = softmax(q . K^T / sqrt(d)) over all N
    keys; `selected` = the sum of p over the tokens of the key tiles the
    selector keeps for the row's tile (select_tiles, `keep` tiles); `special`
    = the sum of p over the special-token keys. Returns (rows [R] token
    indices, selected [R, nh], special [R, nh]) as float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    N, H, d = q.shape
    heads = list(range(H)) if heads is None else list(heads)
    tiles = np.arange(g.n_tiles) if query_tiles is None else np.asarray(query_tiles, dtype=np.int64)
    order, starts, counts = tile_members(g)
    tid = tile_of_token(g)
    rows = np.concatenate([order[starts[t]:starts[t] + counts[t]] for t in tiles]) if len(tiles) else np.zeros(0, np.int64)
    row_tile = tid[rows]
    spec = special_tokens(g)
    sel_mass = np.zeros((len(rows), len(heads)))
    spec_mass = np.zeros((len(rows), len(heads)))
    scale = 1.0 / math.sqrt(d)
    for a, h in enumerate(heads):
        qm = tile_means(q[:, h], g, (order, starts, counts))
        km = tile_means(k[:, h], g, (order, starts, counts))
        sel, _ = select_tiles(qm, km, keep, rows=tiles)
        logits = (q[rows, h] @ k[:, h].T) * scale
        logits -= logits.max(axis=1, keepdims=True)
        p = np.exp(logits)
        p /= p.sum(axis=1, keepdims=True)
        pos = {int(t): i for i, t in enumerate(tiles)}
        for r in range(len(rows)):
            kept = np.flatnonzero(sel[pos[int(row_tile[r])]])
            toks = np.concatenate([order[starts[u]:starts[u] + counts[u]] for u in kept]) if len(kept) else []
            sel_mass[r, a] = p[r, toks].sum()
            spec_mass[r, a] = p[r, spec].sum()
    return rows, sel_mass, spec_mass


# ----------------------------------------------------------------------------
# layer allocation by single-stage linear-conversion error [LC]
# ----------------------------------------------------------------------------
def affine_residual(m: dict, A, b) -> np.ndarray:
    """Mean |A x + b - y|^2 over each group's samples, from its raw moments (READING R23).

    Expands sum |A x + b - y|^2 = tr(A Sxx A^T) + 2 b.(A sx) - 2 tr(A Sxy)
    + n |b|^2 - 2 b.sy + sum |y|^2 and divides by n.
    """
    out = []
    for gi in range(m["n"].shape[0]):
        n = m["n"][gi]
        Ag = np.asarray(A[gi], np.float64)
        bg = np.asarray(b[gi], np.float64)
        total = (np.trace(Ag @ m["sxx"][gi] @ Ag.T) + 2.0 * bg @ (Ag @ m["sx"][gi])
                 - 2.0 * np.trace(Ag @ m["sxy"][gi]) + n * (bg @ bg) - 2.0 * bg @ m["sy"][gi] + m["syy"][gi])
        out.append(total / n)
    return np.array(out)


def allocate_layers(errors, linear_fraction: float) -> np.ndarray:
    """True for the stages that become linear (READING R23)."""
    errors = np.asarray(errors, dtype=np.float64)
    L = errors.shape[0]
    count = int(np.floor(linear_fraction * L + 0.5))
    order = np.argsort(errors, kind="stable")   # ties keep the lower index first
    linear = np.zeros(L, dtype=bool)
    linear[order[:count]] = True
    return linear

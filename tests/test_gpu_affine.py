"""GPU parity of the closed-form centred affine fit (zebra_affine_moments,
zebra_affine_solve), the single-stage conversion error (zebra_affine_residual)
and the layer allocation (zebra_allocate_layers) with the oracle's
affine_moments / affine_solve / affine_residual / allocate_layers.

Page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to Many Views",
section "A closed-form fit avoids retraining from scratch". Moments are float64
sums of products of fp32 or bf16 inputs (exact in float64), so they match the
oracle to rounding-order level; A and b are solved in float64 and stored as
float32.
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

D = 64
KEYS = ("n", "sx", "sy", "sxx", "sxy", "syy")


def _split(buf, groups):
    m = buf.cpu().numpy().reshape(groups, zb.ZEBRA_AFFINE_GROUP_DOUBLES)
    return {"n": m[:, 0], "sx": m[:, 1:1 + D], "sy": m[:, 1 + D:1 + 2 * D],
            "sxx": m[:, 1 + 2 * D:1 + 2 * D + D * D].reshape(groups, D, D),
            "sxy": m[:, 1 + 2 * D + D * D:1 + 2 * D + 2 * D * D].reshape(groups, D, D),
            "syy": m[:, 1 + 2 * D + 2 * D * D]}


def _moments(g, x_d, y_d, per_head, m=None):
    zg = ph.zgeom(g)
    if m is None:
        m = zb.affine_moments_buffer(zg, per_head)
    ws = zb.workspace(zg, zb.ZEBRA_OP_AFFINE)
    zb.zebra_affine_moments(zg, x_d, y_d, m, ws, per_head)
    return m


def _solve(g, m, lam, per_head):
    zg = ph.zgeom(g)
    A = torch.empty((g.heads, D, D), dtype=torch.float32, device="cuda")
    b = torch.empty((g.heads, D), dtype=torch.float32, device="cuda")
    zb.zebra_affine_solve(zg, m, lam, A, b, per_head)
    torch.cuda.synchronize()
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    return A.cpu().numpy().astype(np.float64), b.cpu().numpy().astype(np.float64)


def _samples(g, seed, dtype):
    r = np.random.default_rng(seed)
    shp = (g.n_tokens, g.heads, D)
    x = r.standard_normal(shp).astype(np.float32) + r.standard_normal(D).astype(np.float32)
    y = 0.5 * x[..., ::-1] + r.standard_normal(shp).astype(np.float32) + 1.0
    if dtype == "bf16":
        x, y = synth.round_to_bf16(x), synth.round_to_bf16(y)
    return x, y


@pytest.mark.parametrize("per_head", [False, True], ids=["pooled", "per_head"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_moments_and_solve_match_oracle(per_head, dtype):
    g = Geom(4, 16, 16, 2)
    x, y = _samples(g, 20, dtype)
    m = _moments(g, ph.dev(x, dtype), ph.dev(y, dtype), per_head)
    torch.cuda.synchronize()
    groups = g.heads if per_head else 1
    got = _split(m, groups)
    want = oracle.affine_moments(x, y, per_head)
    for key in KEYS:
        np.testing.assert_allclose(got[key], want[key], rtol=1e-11, atol=1e-8, err_msg=key)
    A, b = _solve(g, m, 0.01, per_head)
    Aw, bw = oracle.affine_solve(want, 0.01)
    heads = range(g.heads)
    for h in heads:
        gi = h if per_head else 0
        np.testing.assert_allclose(A[h], Aw[gi], atol=2e-6, rtol=1e-5)
        np.testing.assert_allclose(b[h], bw[gi], atol=2e-6, rtol=1e-5)


def test_accumulation_over_calls_ragged_bf16():
    # two "scenes" of a ragged geometry with a strided layout (x and y as
    # slices of one buffer), added into the same moments; the fit equals the
    # oracle's fit on both scenes together
    g = Geom(6, 21, 13, 3)
    xs, ys = zip(*(_samples(g, s, "bf16") for s in (31, 32)))
    m = None
    for x, y in zip(xs, ys):
        buf = torch.cat([ph.dev(x, "bf16"), ph.dev(y, "bf16")], dim=2)   # [N, H, 128]
        m = _moments(g, buf[..., :D], buf[..., D:], False, m)
    want = oracle.affine_moments_add(oracle.affine_moments(xs[0], ys[0]), oracle.affine_moments(xs[1], ys[1]))
    torch.cuda.synchronize()
    got = _split(m, 1)
    for key in KEYS:
        np.testing.assert_allclose(got[key], want[key], rtol=1e-11, atol=1e-8, err_msg=key)
    A, b = _solve(g, m, 1e-3, False)
    Aw, bw = oracle.affine_solve(want, 1e-3)
    for h in range(g.heads):
        np.testing.assert_allclose(A[h], Aw[0], atol=2e-6, rtol=1e-5)
        np.testing.assert_allclose(b[h], bw[0], atol=2e-6, rtol=1e-5)


def test_medium_size_per_head_bf16():
    # 32 views x 32x32 patches x 16 heads (N = 32,928): many chunks per head
    g = Geom(32, 32, 32, 16)
    x, y = _samples(g, 33, "bf16")
    m = _moments(g, ph.dev(x, "bf16"), ph.dev(y, "bf16"), True)
    A, b = _solve(g, m, 1e-2, True)
    Aw, bw = oracle.affine_fit(x, y, 1e-2, per_head=True)
    np.testing.assert_allclose(A, Aw, atol=2e-6, rtol=1e-5)
    np.testing.assert_allclose(b, bw, atol=2e-6, rtol=1e-5)


def test_singular_system_reports_numeric_error():
    # constant x with lam = 0: C_xx = 0 is not positive definite -> NaN, status
    g = Geom(2, 8, 8, 1)
    x = np.ones((g.n_tokens, 1, D), np.float32)
    y = np.random.default_rng(34).standard_normal((g.n_tokens, 1, D)).astype(np.float32)
    zg = ph.zgeom(g)
    m = _moments(g, ph.dev(x, "f32"), ph.dev(y, "f32"), False)
    A = torch.zeros((1, D, D), dtype=torch.float32, device="cuda")
    b = torch.zeros((1, D), dtype=torch.float32, device="cuda")
    zb.zebra_affine_solve(zg, m, 0.0, A, b, False)
    torch.cuda.synchronize()
    assert zb.zebra_sync_status() == zb.ZEBRA_ERR_NUMERIC
    assert torch.isnan(A).all() and torch.isnan(b).all()
    assert zb.zebra_sync_status() == zb.ZEBRA_OK   # the status word was cleared by the read


def test_fit_of_the_gpu_linear_stage_to_dense_attention():
    # end to end on the tiny fp32 geometry: x = the GPU linear stage without a
    # correction, y = dense softmax attention (the teacher). Linear outputs span
    # a nearly singular covariance, so the ridge term is set relative to the
    # data (1 % of the mean covariance eigenvalue), as a regularised fit needs.
    # The GPU fit matches the oracle's fit of the same samples, and
    # zebra_linear_attn applies the fitted A, b as y = A x + b.
    g = Geom(4, 16, 16, 2)
    zg = ph.zgeom(g)
    r = np.random.default_rng(35)
    q, k, v = (r.standard_normal((g.n_tokens, g.heads, D)).astype(np.float32) for _ in range(3))
    qd, kd, vd = (ph.dev(t, "f32") for t in (q, k, v))
    ws = zb.workspace(zg, zb.ZEBRA_OP_LINEAR, zb.ZEBRA_F32)
    x_d = torch.empty_like(qd)
    zb.zebra_linear_attn(zg, qd, kd, vd, None, None, x_d, ws)
    y_d = torch.nn.functional.scaled_dot_product_attention(
        qd.permute(1, 0, 2)[None].double(), kd.permute(1, 0, 2)[None].double(),
        vd.permute(1, 0, 2)[None].double())[0].permute(1, 0, 2).float().contiguous()
    xh, yh = ph.host(x_d), ph.host(y_d)
    mw = oracle.affine_moments(xh, yh, per_head=True)
    traces = [np.trace(mw["sxx"][h] / mw["n"][h] - np.outer(mw["sx"][h], mw["sx"][h]) / mw["n"][h] ** 2)
              for h in range(g.heads)]
    lam = 1e-2 * min(traces) / D
    m = _moments(g, x_d, y_d, True)
    A, b = _solve(g, m, lam, True)
    Aw, bw = oracle.affine_solve(mw, lam)
    scale = max(1.0, float(np.abs(Aw).max()))
    np.testing.assert_allclose(A, Aw, atol=1e-4 * scale, rtol=1e-4)
    np.testing.assert_allclose(b, bw, atol=1e-4 * scale, rtol=1e-4)
    out = torch.empty_like(qd)
    zb.zebra_linear_attn(zg, qd, kd, vd, torch.from_numpy(A.astype(np.float32)).cuda(),
                         torch.from_numpy(b.astype(np.float32)).cuda(), out, ws)
    torch.cuda.synchronize()
    want = np.einsum("nhj,hij->nhi", xh, A) + b
    np.testing.assert_allclose(ph.host(out), want, atol=1e-4 * scale, rtol=1e-4)


def test_conversion_errors_and_allocation_match_oracle():
    """Section "Linear-centered stages plus tile-sparse stages": stages are ranked
    by the error of converting each alone to linear attention, and the fraction x
    with the lowest errors becomes linear. Six synthetic stages of the tiny
    geometry (Q, K sharpened by a different factor each, so the linear stage
    misses the dense teacher by different amounts): x = the GPU linear stage
    without a correction, y = the dense teacher (the sparse entry point at
    y = 0), one pooled fit per stage. The GPU's errors (from its moments and
    its fitted A, b) match the oracle's affine_residual of the same samples and
    the same A, b, and the allocations for x = 0.5 and 0.7 match
    oracle.allocate_layers on the oracle's errors."""
    g = Geom(4, 16, 16, 2)
    zg = ph.zgeom(g)
    r = np.random.default_rng(36)
    ws_lin = zb.workspace(zg, zb.ZEBRA_OP_LINEAR, zb.ZEBRA_F32)
    ws_sp = zb.workspace(zg, zb.ZEBRA_OP_SPARSE, zb.ZEBRA_F32, 0.0)
    err_gpu, err_want = [], []
    for stage in range(6):
        sharp = 0.4 + 0.35 * stage
        q, k, v = (r.standard_normal((g.n_tokens, g.heads, D)).astype(np.float32) for _ in range(3))
        q *= np.float32(sharp)
        k *= np.float32(sharp)
        qd, kd, vd = (ph.dev(t, "f32") for t in (q, k, v))
        x_d = torch.empty_like(qd)
        y_d = torch.empty_like(qd)
        zb.zebra_linear_attn(zg, qd, kd, vd, None, None, x_d, ws_lin)
        zb.zebra_sparse_attn(zg, qd, kd, vd, 0.0, y_d, ws_sp)           # y = 0: dense softmax teacher
        m = _moments(g, x_d, y_d, False)
        xh, yh = ph.host(x_d), ph.host(y_d)
        mw = oracle.affine_moments(xh, yh)
        lam = 1e-2 * float(np.trace(mw["sxx"][0] / mw["n"][0] - np.outer(mw["sx"][0], mw["sx"][0]) / mw["n"][0] ** 2)) / D
        A, b = _solve(g, m, lam, False)
        At = torch.from_numpy(A.astype(np.float32)).cuda()
        bt = torch.from_numpy(b.astype(np.float32)).cuda()
        e = torch.empty(1, dtype=torch.float64, device="cuda")
        zb.zebra_affine_residual(zg, m, At, bt, e)
        torch.cuda.synchronize()
        assert zb.zebra_sync_status() == zb.ZEBRA_OK
        got = _split(m, 1)
        np.testing.assert_allclose(got["syy"], mw["syy"], rtol=1e-11)
        want = oracle.affine_residual(mw, A[:1], b[:1])
        # the error also equals the direct mean squared error of the corrected samples
        direct = np.mean(np.sum((np.einsum("nhj,ij->nhi", xh, A[0]) + b[0] - yh) ** 2, axis=-1))
        np.testing.assert_allclose(want[0], direct, rtol=1e-9)
        err_gpu.append(float(e.cpu()[0]))
        err_want.append(float(want[0]))
    np.testing.assert_allclose(err_gpu, err_want, rtol=1e-8)
    assert len(set(np.round(err_want, 6))) == 6          # the stages really differ
    for frac in (0.5, 0.7):
        got = zb.zebra_allocate_layers(err_gpu, frac).astype(bool)
        assert (got == oracle.allocate_layers(err_want, frac)).all()

"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/zebra.h, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import linear_global_attention_b200 as zb
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(zb.LIB_PATH):
        from linear_global_attention_b200 import build
        build.build()
    return zb.lib()


def _declared():
    txt = open(os.path.join(ROOT, "include", "zebra.h")).read()
    return re.findall(r"ZEBRA_API\s+[\w\s\*]+?\b(zebra_\w+)\s*\(", txt)


def test_header_declares_the_entry_points():
    names = set(_declared())
    for n in ("zebra_tile_pool", "zebra_tile_select", "zebra_sparse_attn", "zebra_linear_attn",
              "zebra_hybrid_layer", "zebra_workspace_bytes", "zebra_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 10
    raw = ctypes.CDLL(zb.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n


def test_version_and_launch_count(L):
    assert "sm_100a" in zb.zebra_version()
    assert zb.zebra_launch_count() >= 0


@pytest.mark.parametrize("T", [1, 7, 16, 512, 3200, 12800, 25600, 49152])
@pytest.mark.parametrize("y", [0.0, 0.1, 0.5, 0.6, 0.8, 0.875, 0.9, 0.99, 0.9999])
def test_keep_count_matches_oracle(L, y, T):
    assert zb.zebra_keep_count(y, T) == oracle.keep_count(y, T)


def test_keep_count_rejects_bad_y(L):
    assert zb.zebra_keep_count(1.0, 16) == -1
    assert zb.zebra_keep_count(-0.1, 16) == -1
    assert zb.zebra_keep_count(float("nan"), 16) == -1


def _g(**kw):
    base = dict(views=4, grid_h=16, grid_w=16, heads=2)
    base.update(kw)
    return zb.geom(**base)


def test_workspace_bytes(L):
    g = _g()
    for op in range(7):
        assert zb.zebra_workspace_bytes(g, op, zb.ZEBRA_BF16, 0.6) > 0
    bad = _g(head_dim=32)
    with pytest.raises(zb.ZebraError):
        zb.zebra_workspace_bytes(bad, zb.ZEBRA_OP_SPARSE)
    with pytest.raises(zb.ZebraError):
        zb.zebra_workspace_bytes(_g(), 17)


def _sparse(L, g, dtype=zb.ZEBRA_BF16, y=0.6, ptr=4096, ws=4096, nbytes=1 << 40, layout=None):
    p = ctypes.c_void_p(ptr)
    return L.zebra_sparse_attn(ctypes.byref(g) if g is not None else None, dtype, p, p, p, layout, y, None, p,
                               ctypes.c_void_p(ws) if ws else None, nbytes, None)


def test_sparse_argument_errors(L):
    assert _sparse(L, None) == zb.ZEBRA_ERR_INVALID_ARG
    assert _sparse(L, _g(head_dim=128)) == zb.ZEBRA_ERR_UNSUPPORTED
    assert _sparse(L, _g(tile=16)) == zb.ZEBRA_ERR_UNSUPPORTED
    assert _sparse(L, _g(heads=0)) == zb.ZEBRA_ERR_INVALID_ARG
    assert _sparse(L, _g(grid_h=0)) == zb.ZEBRA_ERR_INVALID_ARG
    assert _sparse(L, _g(views=-1)) == zb.ZEBRA_ERR_INVALID_ARG
    assert _sparse(L, _g(n_special=65)) == zb.ZEBRA_ERR_INVALID_ARG
    assert _sparse(L, _g(), y=1.0) == zb.ZEBRA_ERR_INVALID_ARG
    assert _sparse(L, _g(), y=-0.5) == zb.ZEBRA_ERR_INVALID_ARG
    assert _sparse(L, _g(), dtype=7) == zb.ZEBRA_ERR_INVALID_ARG
    assert _sparse(L, _g(), ptr=0) == zb.ZEBRA_ERR_INVALID_ARG          # null q
    assert _sparse(L, _g(), ptr=4100) == zb.ZEBRA_ERR_INVALID_ARG       # misaligned
    assert _sparse(L, _g(), nbytes=16) == zb.ZEBRA_ERR_WORKSPACE
    assert _sparse(L, _g(), ws=0) == zb.ZEBRA_ERR_WORKSPACE
    assert _sparse(L, _g(), ws=4096 + 16) == zb.ZEBRA_ERR_WORKSPACE       # base not 256-byte aligned
    assert "aligned" in zb.zebra_last_error()
    bad_layout = zb.Layout(130, 64)
    assert _sparse(L, _g(), layout=ctypes.byref(bad_layout)) == zb.ZEBRA_ERR_INVALID_ARG
    assert "strides" in zb.zebra_last_error()
    # more tiles than the selector handles
    assert _sparse(L, _g(views=2000, grid_h=64, grid_w=64)) == zb.ZEBRA_ERR_UNSUPPORTED
    # 49,152 tiles x 700 heads x 64 rows: beyond 32-bit TMA row coordinates
    assert _sparse(L, _g(views=768, grid_h=64, grid_w=64, heads=700, n_special=0)) == zb.ZEBRA_ERR_UNSUPPORTED
    assert "2^31" in zb.zebra_last_error()


def test_empty_input_is_a_noop(L):
    # views == 0: nothing to do, no device needed
    assert _sparse(L, _g(views=0), ptr=0, ws=0, nbytes=0) == zb.ZEBRA_OK
    p = ctypes.c_void_p(0)
    g = _g(views=0)
    assert L.zebra_linear_attn(ctypes.byref(g), zb.ZEBRA_BF16, p, p, p, None, None, None, 100.0, 1e-6, p, None, 0,
                               None) == zb.ZEBRA_OK
    assert L.zebra_hybrid_layer(ctypes.byref(g), 0, p, p, p, None, None, 0.0, 100.0, 1e-6, p, None, 0,
                                None) == zb.ZEBRA_OK
    assert L.zebra_tile_pool(ctypes.byref(g), zb.ZEBRA_BF16, p, None, p, None, None, None) == zb.ZEBRA_OK


def test_linear_and_hybrid_argument_errors(L):
    p = ctypes.c_void_p(4096)
    g = _g()
    assert L.zebra_linear_attn(ctypes.byref(g), zb.ZEBRA_BF16, p, p, p, None, None, None, 0.0, 1e-6, p, p, 1 << 40,
                               None) == zb.ZEBRA_ERR_INVALID_ARG   # rope_base 0
    assert L.zebra_linear_attn(ctypes.byref(g), zb.ZEBRA_BF16, p, p, p, None, None, None, 100.0, 1e-6, p, p, 8,
                               None) == zb.ZEBRA_ERR_WORKSPACE
    assert L.zebra_hybrid_layer(ctypes.byref(g), 9, p, p, p, None, None, 0.5, 100.0, 1e-6, p, p, 1 << 40,
                                None) == zb.ZEBRA_ERR_INVALID_ARG  # kind
    assert L.zebra_hybrid_layer(ctypes.byref(g), 1, p, p, p, None, None, 1.5, 100.0, 1e-6, p, p, 1 << 40,
                                None) == zb.ZEBRA_ERR_INVALID_ARG  # y
    assert L.zebra_hybrid_layer(ctypes.byref(g), 1, p, p, p, None, None, 0.5, 100.0, 1e-6, p, p, 8,
                                None) == zb.ZEBRA_ERR_WORKSPACE


def test_select_argument_errors(L):
    p = ctypes.c_void_p(4096)
    g = _g()
    k = ctypes.c_int32(0)
    assert L.zebra_tile_select(ctypes.byref(g), p, p, 1.0, p, None, ctypes.byref(k), p, 1 << 40,
                               None) == zb.ZEBRA_ERR_INVALID_ARG
    assert L.zebra_tile_select(ctypes.byref(g), p, p, 0.6, None, None, ctypes.byref(k), p, 1 << 40,
                               None) == zb.ZEBRA_ERR_INVALID_ARG
    assert k.value == 7   # keep count is reported before the mask check
    assert L.zebra_tile_select(ctypes.byref(g), p, p, 0.6, p, None, ctypes.byref(k), p, 4,
                               None) == zb.ZEBRA_ERR_WORKSPACE


def test_no_gpu_gives_a_cuda_error_not_a_crash(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _sparse(L, _g()) == zb.ZEBRA_ERR_CUDA
    assert "CUDA" in zb.zebra_last_error() or "device" in zb.zebra_last_error()


def test_affine_argument_errors(L):
    p = ctypes.c_void_p(4096)
    g = _g()
    big = 1 << 40

    def moments(ptr=p, per_head=0, nbytes=big, xptr=p, layout=None, dtype=zb.ZEBRA_BF16):
        return L.zebra_affine_moments(ctypes.byref(g), dtype, xptr, p, layout, per_head, ptr, p, nbytes, None)

    assert moments(ptr=None) == zb.ZEBRA_ERR_INVALID_ARG                      # moments null
    assert moments(ptr=ctypes.c_void_p(4100)) == zb.ZEBRA_ERR_INVALID_ARG     # moments misaligned
    assert moments(per_head=2) == zb.ZEBRA_ERR_INVALID_ARG
    assert moments(xptr=ctypes.c_void_p(4104)) == zb.ZEBRA_ERR_INVALID_ARG    # x misaligned
    assert moments(dtype=5) == zb.ZEBRA_ERR_INVALID_ARG
    assert moments(layout=ctypes.byref(zb.Layout(130, 64))) == zb.ZEBRA_ERR_INVALID_ARG
    assert moments(nbytes=64) == zb.ZEBRA_ERR_WORKSPACE
    e = _g(views=0)
    assert L.zebra_affine_moments(ctypes.byref(e), zb.ZEBRA_BF16, None, None, None, 0, p, None, 0,
                                  None) == zb.ZEBRA_OK                        # empty: nothing to add
    for lam in (-1.0, float("nan"), float("inf")):
        assert L.zebra_affine_solve(ctypes.byref(g), p, 0, lam, p, p, None) == zb.ZEBRA_ERR_INVALID_ARG
    assert L.zebra_affine_solve(ctypes.byref(g), None, 0, 0.1, p, p, None) == zb.ZEBRA_ERR_INVALID_ARG
    assert L.zebra_affine_solve(ctypes.byref(g), p, 0, 0.1, None, p, None) == zb.ZEBRA_ERR_INVALID_ARG
    assert L.zebra_affine_solve(ctypes.byref(g), p, 3, 0.1, p, p, None) == zb.ZEBRA_ERR_INVALID_ARG


def _hybrid(L, g, kind, y=0.8, ptr=4096):
    p = ctypes.c_void_p(ptr)
    return L.zebra_hybrid_layer(ctypes.byref(g), kind, p, p, p, None, None, y, 100.0, 1e-6, p, p, 1 << 40, None)


@pytest.mark.parametrize("kind", [zb.ZEBRA_LAYER_SPARSE, zb.ZEBRA_LAYER_DENSE])
def test_hybrid_layer_rejects_32bit_tma_overflow(L, kind):
    # 49,152 tiles x 700 heads x 64 rows: beyond 32-bit TMA row coordinates, refused before any launch
    assert _hybrid(L, _g(views=768, grid_h=64, grid_w=64, heads=700, n_special=0), kind) == zb.ZEBRA_ERR_UNSUPPORTED
    assert "2^31" in zb.zebra_last_error()


def test_hybrid_layer_argument_errors(L):
    assert _hybrid(L, _g(), 7) == zb.ZEBRA_ERR_INVALID_ARG                       # unknown kind
    assert _hybrid(L, _g(), zb.ZEBRA_LAYER_SPARSE, y=1.0) == zb.ZEBRA_ERR_INVALID_ARG
    assert _hybrid(L, _g(), zb.ZEBRA_LAYER_LINEAR, ptr=4100) == zb.ZEBRA_ERR_INVALID_ARG
    # more tiles than the selector handles
    assert _hybrid(L, _g(views=2000, grid_h=64, grid_w=64), zb.ZEBRA_LAYER_SPARSE) == zb.ZEBRA_ERR_UNSUPPORTED


def test_noalloc_shares_the_argument_checks(L):
    p = ctypes.c_void_p(4096)

    def call(g, layout=None, ptr=p):
        return L.zebra_linear_attn_noalloc(ctypes.byref(g), zb.ZEBRA_BF16, ptr, ptr, ptr, layout, None, None,
                                           100.0, 1e-6, ptr, None)

    # the same statuses as zebra_linear_attn for the same bad inputs
    for g, code in ((_g(head_dim=32), zb.ZEBRA_ERR_UNSUPPORTED), (_g(grid_h=5000), zb.ZEBRA_ERR_UNSUPPORTED),
                    (_g(heads=0), zb.ZEBRA_ERR_INVALID_ARG), (_g(views=1 << 30, grid_h=64, grid_w=64),
                                                              zb.ZEBRA_ERR_UNSUPPORTED)):
        assert call(g) == code
        assert L.zebra_linear_attn(ctypes.byref(g), zb.ZEBRA_BF16, p, p, p, None, None, None, 100.0, 1e-6, p, p,
                                   1 << 40, None) == code
    assert call(_g(), layout=ctypes.byref(zb.Layout(130, 64))) == zb.ZEBRA_ERR_INVALID_ARG
    assert call(_g(), ptr=ctypes.c_void_p(4100)) == zb.ZEBRA_ERR_INVALID_ARG


@pytest.mark.parametrize("frac", [0.0, 0.3, 0.5, 0.7, 1.0])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_allocate_layers_matches_oracle(L, frac, seed):
    import numpy as np
    rng = np.random.default_rng(seed)
    err = rng.integers(0, 6, 24).astype(np.float64)      # many ties
    err[rng.integers(0, 24, 2)] = np.nan                   # NaN ranks last
    got = zb.zebra_allocate_layers(err, frac).astype(bool)
    assert (got == oracle.allocate_layers(err, frac)).all()
    assert got.sum() == int(np.floor(frac * 24 + 0.5))


def test_allocate_layers_rejects_bad_arguments(L):
    import numpy as np
    assert L.zebra_allocate_layers(None, 3, 0.5, None) == -1
    e = np.zeros(3)
    out = np.zeros(3, np.int32)
    assert L.zebra_allocate_layers(e.ctypes.data_as(ctypes.c_void_p), 3, 1.5,
                                   out.ctypes.data_as(ctypes.c_void_p)) == -1
    assert L.zebra_allocate_layers(None, 0, 0.5, None) == 0


def test_affine_residual_argument_errors(L):
    p = ctypes.c_void_p(4096)
    g = _g()
    assert L.zebra_affine_residual(ctypes.byref(g), None, 0, p, p, p, None) == zb.ZEBRA_ERR_INVALID_ARG
    assert L.zebra_affine_residual(ctypes.byref(g), p, 2, p, p, p, None) == zb.ZEBRA_ERR_INVALID_ARG
    assert L.zebra_affine_residual(ctypes.byref(g), p, 0, p, p, ctypes.c_void_p(4100), None) == zb.ZEBRA_ERR_INVALID_ARG
    assert L.zebra_affine_residual(ctypes.byref(g), p, 0, None, p, p, None) == zb.ZEBRA_ERR_INVALID_ARG

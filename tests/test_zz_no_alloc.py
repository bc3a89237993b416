"""GPU test of zebra_linear_attn_noalloc, the linear-stage entry point for
callers that cannot allocate device memory (its scratch is a built-in device
array instead of a caller workspace).

Two calls in a row on different inputs are compared with zebra_linear_attn,
the workspace-based entry point. Below the size at which the chunk partials
fill the built-in array the two entry points sum in the same order, so the
outputs must be bit-identical; above it (128 views) the chunks grow and the
outputs must agree within the bf16 tolerance of the parity tests. The second
call of each pair checks that nothing left in the shared scratch array by the
first call leaks into its result. The file name makes pytest collect it last;
it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_global_attention_b200 as zb
import synth
from tests import parity_helpers as ph

pytestmark = pytest.mark.gpu


def _inputs(seed, views):
    w = synth.custom(views, 37, 37, 16, seed=seed, recipe="iid", dtype="bf16")
    q, k, v = synth.qkv(w)
    A, b = synth.affine(16, seed)
    return w, q, k, v, A, b


@pytest.mark.parametrize("views,exact", [(6, True), (128, False)], ids=["same_chunks", "grown_chunks"])
def test_noalloc_matches_workspace_entry_point_twice(views, exact):
    dtype = "bf16"
    results = []
    for seed in (31, 32):                       # two calls in a row, different inputs
        w, q, k, v, A, b = _inputs(seed, views)
        g = zb.geom(w.views, w.grid_h, w.grid_w, w.heads)
        qd, kd, vd = ph.dev(q, dtype), ph.dev(k, dtype), ph.dev(v, dtype)
        At, bt = torch.from_numpy(A).cuda(), torch.from_numpy(b).cuda()
        ref = torch.empty_like(qd)
        ws = zb.workspace(g, zb.ZEBRA_OP_LINEAR, zb.ZEBRA_BF16)
        zb.zebra_linear_attn(g, qd, kd, vd, At, bt, ref, ws)
        out = torch.full_like(qd, float("nan"))
        zb.zebra_linear_attn_noalloc(g, qd, kd, vd, At, bt, out)
        torch.cuda.synchronize()
        assert zb.zebra_sync_status() == zb.ZEBRA_OK
        got, want = ph.host(out), ph.host(ref)
        assert np.isfinite(got).all()
        ph.assert_close(got, want, dtype, f"noalloc vs workspace entry point, {views} views, seed {seed}")
        if exact:
            assert torch.equal(out, ref), "same chunks must give bit-identical outputs"
        results.append(got)
    assert not np.array_equal(results[0], results[1])


def test_noalloc_rejects_oversized_geometry():
    # 1024 heads need 1024 x 64 x 65 x 4 bytes of state alone: more than the built-in area
    g = zb.geom(1, 8, 8, 1024)
    x = torch.empty((g.n_tokens, 1024, 64), dtype=torch.bfloat16, device="cuda")
    rc = zb.lib().zebra_linear_attn_noalloc(ctypes.byref(g), zb.ZEBRA_BF16, ctypes.c_void_p(x.data_ptr()),
                                            ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(x.data_ptr()), None,
                                            None, None, 100.0, 1e-6, ctypes.c_void_p(x.data_ptr()), None)
    assert rc == zb.ZEBRA_ERR_UNSUPPORTED
    assert "16 MiB" in zb.zebra_last_error()

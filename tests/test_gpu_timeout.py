"""The bounded-wait error paths of the tcgen05 sparse and linear-state kernels, exercised without a fault.

The test hook zebra_debug_inject makes the kernel's copy producer stop before
block 2 of every query tile's block stream and shortens every wait to 5 ms.
The tensor-core warp's wait for block 2's keys then runs out: the kernel must
record ZEBRA_ERR_TIMEOUT, drain its copies and MMAs, free its tensor memory and
exit, and zebra_sync_status must report the timeout. After the hook is turned
off, the same call on the same inputs must match the oracle again (the context
stays usable and nothing is left behind). Every wait in the kernel is bounded,
so nothing here can hang the GPU.

The same hook makes the linear stage's state kernel leave out the MMAs of
block 1 of every token chunk; its wait for their completion runs out the same
way.
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


def test_wait_timeout_reports_and_recovers():
    g = Geom(3, 16, 16, 2)                 # 12 tiles; every query tile streams >= 3 blocks
    rng = np.random.default_rng(23)
    q, k, v = (synth.round_to_bf16(rng.standard_normal((g.n_tokens, 2, 64)).astype(np.float32))
               for _ in range(3))
    y = 0.5
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    try:
        zb.zebra_debug_inject(2, 5_000_000)
        ph.run_sparse(g, q, k, v, y, "bf16")
        assert zb.zebra_sync_status() == zb.ZEBRA_ERR_TIMEOUT
        assert "wait" in zb.zebra_last_error()
    finally:
        zb.zebra_debug_inject(-1, 0)
    assert zb.zebra_sync_status() == zb.ZEBRA_OK          # the status word was cleared by the read
    out = ph.host(ph.run_sparse(g, q, k, v, y, "bf16"))
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    keep = oracle.keep_count(y, g.n_tiles)
    sel, _, _, _ = ph.run_select(g, q, k, y, "bf16")
    near = ph.check_selection(g, q, k, keep, sel, what="after timeout")
    want = oracle.sparse_stage_full(q, k, v, g, keep)
    tid = oracle.tile_of_token(g)
    for h in range(g.heads):
        ok = ~np.isin(tid, near[h])
        ph.assert_close(out[ok, h], want[ok, h], "bf16", f"after timeout head {h}")


def test_linear_wait_timeout_reports_and_recovers():
    g = Geom(2, 16, 16, 2)                 # 522 tokens: one chunk of 9 blocks of 64
    rng = np.random.default_rng(29)
    q, k, v = (synth.round_to_bf16(rng.standard_normal((g.n_tokens, 2, 64)).astype(np.float32))
               for _ in range(3))
    A, b = synth.affine(g.heads, 29)
    zg = ph.zgeom(g)
    qd, kd, vd = ph.dev(q, "bf16"), ph.dev(k, "bf16"), ph.dev(v, "bf16")
    At, bt = torch.from_numpy(A).cuda(), torch.from_numpy(b).cuda()
    out = torch.empty_like(qd)
    ws = zb.workspace(zg, zb.ZEBRA_OP_LINEAR, zb.ZEBRA_BF16)
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    try:
        zb.zebra_debug_inject(1, 5_000_000)
        zb.zebra_linear_attn(zg, qd, kd, vd, At, bt, out, ws)
        assert zb.zebra_sync_status() == zb.ZEBRA_ERR_TIMEOUT
        assert "wait" in zb.zebra_last_error()
    finally:
        zb.zebra_debug_inject(-1, 0)
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    zb.zebra_linear_attn(zg, qd, kd, vd, At, bt, out, ws)
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    ph.assert_close(ph.host(out), oracle.linear_stage(q, k, v, g, A, b), "bf16", "linear after timeout")

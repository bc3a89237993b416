"""GPU parity at the headline size: 1,024 views of 37x37 patches plus 5 special
tokens (N = 1,406,976), 16 heads, the launch configuration the benchmark's
stacked layers use (Q/K/V as strided slices of one [N, 3*1024] projection
buffer; sparse stage at y = 0.8, i.e. 5,120 of 25,600 key tiles kept).

The oracle evaluates sampled outputs: whole query tiles (and special-token
rows) of the sparse stage, and sampled token rows of the linear stage, for a
few heads, from the same seeded inputs. Selections of the sampled rows must be
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

W = synth.custom(1024, 37, 37, 16, seed=4104, recipe="iid", dtype="bf16", name="fullsize_v1024")
G = Geom(1024, 37, 37, 16)
HEADS = [0, 9]


@pytest.fixture(scope="module")
def qkv():
    q, k, v = synth.qkv(W)
    return q, k, v


@pytest.fixture(scope="module")
def dev_qkv(qkv):
    """Q/K/V packed side by side like the stacked layer's projection output."""
    N, H = G.n_tokens, G.heads
    buf = torch.empty((N, 3 * H * 64), dtype=torch.bfloat16, device="cuda")
    for i, x in enumerate(qkv):
        buf[:, i * H * 64:(i + 1) * H * 64] = torch.from_numpy(x.reshape(N, H * 64)).to(torch.bfloat16).cuda()
    views = tuple(buf[:, i * H * 64:(i + 1) * H * 64].view(N, H, 64) for i in range(3))
    return buf, views


def test_sparse_stage_full_size_sampled(qkv, dev_qkv):
    q, k, v = qkv
    _, (qd, kd, vd) = dev_qkv
    zg = ph.zgeom(G)
    y = 0.8
    keep = oracle.keep_count(y, G.n_tiles)
    assert keep == 5120
    out = torch.empty((G.n_tokens, G.heads, 64), dtype=torch.bfloat16, device="cuda")
    ws = zb.workspace(zg, zb.ZEBRA_OP_SPARSE, zb.ZEBRA_BF16, y)
    zb.zebra_sparse_attn(zg, qd, kd, vd, y, out, ws)
    torch.cuda.synchronize()
    assert zb.zebra_sync_status() == zb.ZEBRA_OK
    del ws
    rng = np.random.default_rng(11)
    tiles = np.sort(rng.choice(G.n_tiles, 3, replace=False))
    specials = np.sort(rng.choice(oracle.special_tokens(G), 2, replace=False))
    rows, want, sel, gaps = oracle.sparse_stage(q, k, v, G, keep, query_tiles=tiles, special_rows=specials,
                                                heads=HEADS)
    got = out[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    tid = oracle.tile_of_token(G)
    for h in HEADS:
        near_tiles = tiles[gaps[h] < oracle.NEAR_TIE_REL_GAP]
        ph.record_near_ties(f"full-size sparse head {h}", len(tiles), len(near_tiles))
        ok = ~np.isin(tid[rows], near_tiles)
        ph.assert_close(got[ok, h], want[ok, h], "bf16", f"full-size sparse head {h}")
    # selections of the sampled query tiles are bit-exact outside near-ties
    qm = torch.empty((G.heads, G.n_tiles, 64), device="cuda")
    km = torch.empty_like(qm)
    zb.zebra_tile_pool(zg, qd, qm)
    zb.zebra_tile_pool(zg, kd, km)
    mask = torch.empty((G.heads, G.n_tiles, zg.mask_words), dtype=torch.int32, device="cuda")
    ws = zb.workspace(zg, zb.ZEBRA_OP_SELECT, zb.ZEBRA_BF16, y)
    zb.zebra_tile_select(zg, qm, km, y, mask, None, ws)
    torch.cuda.synchronize()
    gsel = ph.unpack_mask(mask[:, torch.from_numpy(tiles).cuda()], G.n_tiles)
    for h in HEADS:
        nt = gaps[h] < oracle.NEAR_TIE_REL_GAP
        assert (gsel[h].sum(1) == keep).all()
        assert not ((gsel[h] != sel[h]).any(1) & ~nt).any(), f"head {h}: selection differs outside near-ties"


def test_linear_stage_full_size_sampled(qkv, dev_qkv):
    q, k, v = qkv
    _, (qd, kd, vd) = dev_qkv
    zg = ph.zgeom(G)
    A, b = synth.affine(G.heads, 4104)
    out = torch.empty((G.n_tokens, G.heads, 64), dtype=torch.bfloat16, device="cuda")
    ws = zb.workspace(zg, zb.ZEBRA_OP_LINEAR)
    zb.zebra_linear_attn(zg, qd, kd, vd, torch.from_numpy(A).cuda(), torch.from_numpy(b).cuda(), out, ws)
    torch.cuda.synchronize()
    rng = np.random.default_rng(12)
    rows = np.sort(rng.choice(G.n_tokens, 3000, replace=False))
    want = oracle.linear_stage(q, k, v, G, A, b, rows=rows, heads=HEADS)
    got = out[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    for h in HEADS:
        ph.assert_close(got[:, h], want[:, h], "bf16", f"full-size linear head {h}")

"""Inputs of the small stacked-layer parity cases, chosen so that the attention
term dominates the layer's output.

With the benchmark's weights (W ~ N(0, 0.02^2)) the residual x carries more
than 99% of x_out = x + Attn(..) W_o^T, so a comparison of x_out at the bf16
tolerance cannot see the attention. Here x is small (0.1 N(0,1)), the QKV
projection brings q, k to an RMS of about 3 and v to about 1 (so dropping the
Q/K normalisation changes the logits ninefold), and W_o is large enough that
|x_out - x| / |x_out| >= 0.9 on the oracle; every test that uses these inputs
asserts that ratio.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth
from oracle import Geom

GEOM = Geom(5, 13, 11, 4)      # partial edge tiles (13 = 8 + 5, 11 = 8 + 3), 20 tiles
Y = 0.6                        # keeps 8 of 20 key tiles per query tile
MIN_ATTN_SHARE = 0.9


def small_case(seed: int = 17):
    g = GEOM
    D = g.heads * 64
    rng = np.random.default_rng(seed)
    x = synth.round_to_bf16((0.1 * rng.standard_normal((g.n_tokens, D))).astype(np.float32))
    scale = np.concatenate([np.full(2 * D, 30.0), np.full(D, 10.0)]) / np.sqrt(D)   # q, k rows; v rows
    wqkv = synth.round_to_bf16((rng.standard_normal((3 * D, D)) * scale[:, None]).astype(np.float32))
    wo = synth.round_to_bf16((8.0 / np.sqrt(D) * rng.standard_normal((D, D))).astype(np.float32))
    A, b = synth.affine(g.heads, seed)
    return x, wqkv, wo, A, b


def attention_share(x, x_out) -> float:
    """|x_out - x| / |x_out|: the attention term's share of the output norm."""
    return float(np.linalg.norm(x_out - x) / np.linalg.norm(x_out))


def qkv_bf16(qkv):
    """The kernel's storage of the QKV projection: fp32 accumulation rounded to bf16."""
    return synth.round_to_bf16(np.asarray(qkv, np.float32))


def oracle_out(kind: str, mod=oracle, seed: int = 17):
    """(x, the oracle's x_out) with the projection taken in the kernel's storage
    precision (bf16), so that both sides select key tiles from the same values."""
    x, wqkv, wo, A, b = small_case(seed)
    keep = mod.keep_count(Y, GEOM.n_tiles)
    return x, mod.hybrid_layer(x, wqkv, wo, kind, GEOM, A=A, b=b, keep=keep, qkv_round=qkv_bf16)

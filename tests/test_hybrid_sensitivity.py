"""The small stacked-layer parity cases can see the attention they check.

CPU only. For each layer kind, a plausible mistake is planted in a private copy
of the oracle (Q/K normalisation dropped, 2D rotation dropped, the attention
term dropped, ...) and the mistaken output is compared with the true oracle on
the inputs the GPU test uses: it must fail the bf16 acceptance bar that the GPU
test applies. A kernel that made the same mistake would therefore fail that
test. The real oracle module is never modified.
"""
import importlib.util
import sys

import numpy as np
import pytest

import oracle
import oracle.zebra_oracle as zo
from tests import hybrid_cases as hc

TOL = (2e-2, 5e-3)       # max |err|, relative L2: the bf16 bar of the GPU parity tests
SRC = open(zo.__file__).read()


def _mutant(edits):
    src = SRC
    for old, new in edits:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    spec = importlib.util.spec_from_loader("oracle_hybrid_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    sys.modules["oracle_hybrid_mutant"] = mod
    exec(compile(src, "oracle_hybrid_mutant.py", "exec"), mod.__dict__)
    return mod


def _fails_bar(got, want) -> bool:
    d = got - want
    return float(np.abs(d).max()) > TOL[0] or float(np.linalg.norm(d) / np.linalg.norm(want)) > TOL[1]


QK_NORM = ("qn = rope_2d(rms_norm(q, eps), g, rope_base)\n        kn = rope_2d(rms_norm(k, eps), g, rope_base)",)
MISTAKES = {
    "sparse/dense: Q/K RMS norm dropped": (("sparse", "dense"), [(QK_NORM[0], "qn = rope_2d(q, g, rope_base)\n"
                                                                 "        kn = rope_2d(k, g, rope_base)")]),
    "sparse/dense: 2D rotation dropped": (("sparse", "dense"), [(QK_NORM[0], "qn = rms_norm(q, eps)\n"
                                                                 "        kn = rms_norm(k, eps)")]),
    "sparse/dense: rotation on V too": (("sparse", "dense"), [
        ("o = sparse_stage_full(qn, kn, v, g, keep)", "o = sparse_stage_full(qn, kn, rope_2d(v, g, rope_base), g, keep)"),
        ("dense_attention(qn[:, h], kn[:, h], v[:, h])", "dense_attention(qn[:, h], kn[:, h], rope_2d(v, g, rope_base)[:, h])")]),
    "linear: Q/K RMS norm dropped": (("linear",), [("return phi(rope_2d(rms_norm(x, eps), g, rope_base, rows=rows))",
                                                     "return phi(rope_2d(x, g, rope_base, rows=rows))")]),
    "linear: 2D rotation dropped": (("linear",), [("return phi(rope_2d(rms_norm(x, eps), g, rope_base, rows=rows))",
                                                    "return phi(rms_norm(x, eps))")]),
    "linear: affine correction dropped": (("linear",), [
        ("out[:, h] = o @ np.asarray(A[h], np.float64).T + np.asarray(b[h], np.float64)", "out[:, h] = o")]),
    "attention term dropped": (("linear", "sparse", "dense"), [
        ("return x + o.reshape(N, -1) @ np.asarray(w_o, np.float64).T",
         "return x + 0.0 * (o.reshape(N, -1) @ np.asarray(w_o, np.float64).T)")]),
    "output projection transposed": (("linear", "sparse", "dense"), [
        ("return x + o.reshape(N, -1) @ np.asarray(w_o, np.float64).T",
         "return x + o.reshape(N, -1) @ np.asarray(w_o, np.float64)")]),
}


@pytest.mark.parametrize("kind", ["linear", "sparse", "dense"])
def test_attention_dominates_the_output(kind):
    x, want = hc.oracle_out(kind)
    assert hc.attention_share(x, want) >= hc.MIN_ATTN_SHARE


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_planted_mistake_fails_the_bar(name):
    kinds, edits = MISTAKES[name]
    mod = _mutant(edits)
    for kind in kinds:
        _, want = hc.oracle_out(kind)
        _, got = hc.oracle_out(kind, mod=mod)
        assert _fails_bar(got, want), f"{name} ({kind}) would pass the bf16 bar"


def test_sparse_layer_differs_from_dense_beyond_the_bar():
    # the sparse case keeps 8 of 20 tiles: a kernel that ignored the selection would fail
    _, sparse = hc.oracle_out("sparse")
    _, dense = hc.oracle_out("dense")
    assert _fails_bar(sparse, dense)

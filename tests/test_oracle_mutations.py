"""Planted mistakes in the oracle must be caught by the pins.

Each case edits one line of a private copy of the oracle's source (a dropped
term, a wrong sign or index, a transposed operand), loads the copy as a
separate module, points the pin tests at it and checks that at least one of
the listed pins fails. The real oracle module is never modified. CPU only.
"""
import importlib.util
import os
import sys
import types

import pytest

import oracle.zebra_oracle as zo
from tests import test_oracle_affine as affine_pins
from tests import test_oracle_coverage as coverage_pins
from tests import test_oracle_pins as pins

SRC = open(zo.__file__).read()


def _mutant(old: str, new: str) -> types.ModuleType:
    assert SRC.count(old) >= 1, old
    spec = importlib.util.spec_from_loader("oracle_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    sys.modules["oracle_mutant"] = mod
    exec(compile(SRC.replace(old, new), "oracle_mutant.py", "exec"), mod.__dict__)
    return mod


def _fails(pin_calls, mod, monkeypatch):
    monkeypatch.setattr(pins, "oracle", mod)
    monkeypatch.setattr(affine_pins, "oracle", mod)
    monkeypatch.setattr(coverage_pins, "oracle", mod)
    for call in pin_calls:
        try:
            call()
        except (AssertionError, ValueError, IndexError):
            return True
    return False


G = pins.Geom
MUTATIONS = [
    ("drop landmark ln(m)", "np.log(counts[lm])", "np.zeros(len(lm))",
     [lambda: pins.test_constant_keys_give_the_global_value_mean(3)]),
    ("drop own-landmark ln(m)", "* scale + math.log(m))", "* scale)",
     [lambda: pins.test_constant_keys_give_the_global_value_mean(3)]),
    ("own tile counted twice", "if not sel[a, u] and u != t]", "if not sel[a, u]]",
     [lambda: pins.test_constant_keys_give_the_global_value_mean(3)]),
    ("self key dropped", "extra_logits = [self_logit[:, None]]", "extra_logits = [self_logit[:, None] - 1e9]",
     [lambda: pins.test_constant_keys_give_the_global_value_mean(3)]),
    ("special keys dropped", "keys = np.concatenate([kh[exact], k_spec, k_mean[lm]])",
     "keys = np.concatenate([kh[exact], k_spec - 1e6, k_mean[lm]])",
     [lambda: pins.test_y0_equals_dense_softmax_attention(G(4, 16, 16, 2))]),
    ("means over 64 instead of n_u", "return sums / counts[:, None]", "return sums / 64.0",
     [pins.test_tile_means_against_direct_loops]),
    ("selector keeps the lowest scores", 'order = np.argsort(-s, axis=1, kind="stable")',
     'order = np.argsort(s, axis=1, kind="stable")',
     [lambda: pins.test_selector_against_exhaustive_subset_search(0)]),
    ("selector ties to the highest index", 'order = np.argsort(-s, axis=1, kind="stable")',
     'order = (s.shape[1] - 1 - np.argsort(-s[:, ::-1], axis=1, kind="stable"))',
     [lambda: pins.test_selector_against_exhaustive_subset_search(s) for s in range(6)]),
    ("wrong softmax scale", "scale = 1.0 / math.sqrt(d)", "scale = 1.0 / d",
     [lambda: pins.test_y0_equals_dense_softmax_attention(G(4, 16, 16, 2))]),
    ("keep count floor", "k = math.ceil((1.0 - y) * n_tiles - 1e-6)", "k = math.floor((1.0 - y) * n_tiles)",
     [pins.test_keep_count_rule]),
    ("rope sign", "out[..., off:off + quarter] = a * c - b * s", "out[..., off:off + quarter] = a * c + b * s",
     [pins.test_rope_matches_complex_rotation_and_base_100]),
    ("rope frequency exponent", "theta = base ** (-2.0 * np.arange(quarter) / half)",
     "theta = base ** (-2.0 * np.arange(quarter) / d)",
     [pins.test_rope_matches_complex_rotation_and_base_100]),
    ("rope row/col swapped", "for off, pos in ((0, row), (half, col)):", "for off, pos in ((0, col), (half, row)):",
     [pins.test_rope_matches_complex_rotation_and_base_100]),
    ("rms uses sum", "np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)",
     "np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)",
     [pins.test_rms_norm_unit_rms_and_scale_invariance]),
    ("linear normaliser dropped", "o = (fq @ S) / (fq @ z)[:, None]", "o = (fq @ S)",
     [pins.test_linear_stage_equals_explicit_kernel_product]),
    ("affine transposed", "out[:, h] = o @ np.asarray(A[h], np.float64).T + np.asarray(b[h], np.float64)",
     "out[:, h] = o @ np.asarray(A[h], np.float64) + np.asarray(b[h], np.float64)",
     [pins.test_linear_stage_constant_features_closed_form]),
    ("affine bias dropped", "out[:, h] = o @ np.asarray(A[h], np.float64).T + np.asarray(b[h], np.float64)",
     "out[:, h] = o @ np.asarray(A[h], np.float64).T",
     [pins.test_linear_stage_constant_features_closed_form]),
    ("phi over tokens", "e = np.exp(x - x.max(axis=-1, keepdims=True))\n    return e / e.sum(axis=-1, keepdims=True)",
     "e = np.exp(x - x.max(axis=-1, keepdims=True))\n    return e / e.sum(axis=0, keepdims=True)",
     [pins.test_phi_is_a_channel_softmax]),
    ("output projection transposed", "return x + o.reshape(N, -1) @ np.asarray(w_o, np.float64).T",
     "return x + o.reshape(N, -1) @ np.asarray(w_o, np.float64)",
     [pins.test_hybrid_dense_layer_against_library_composition]),
    ("q/k swapped in split", "return tuple(qkv[:, i * D:(i + 1) * D].reshape(N, heads, d) for i in range(3))",
     "return tuple(qkv[:, j * D:(j + 1) * D].reshape(N, heads, d) for j in (1, 0, 2))",
     [pins.test_hybrid_dense_layer_against_library_composition]),
    ("tile column index uses grid rows", "(row // g.tile) * g.tile_cols + (col // g.tile)",
     "(row // g.tile) * g.tile_rows + (col // g.tile)",
     [pins.test_tile_index_is_row_major_and_views_do_not_mix]),
    ("affine covariance not centred", 'cxx = m["sxx"][gi] / n - np.outer(mu_x, mu_x)', 'cxx = m["sxx"][gi] / n',
     [affine_pins.test_noise_free_recovery_per_head]),
    ("affine A transposed", "A = a_t.T", "A = a_t",
     [affine_pins.test_noise_free_recovery_per_head]),
    ("affine bias ignores mean of x", "out_b.append(mu_y - A @ mu_x)", "out_b.append(mu_y)",
     [affine_pins.test_noise_free_recovery_per_head]),
    ("affine ridge term dropped", "cxx + lam * np.eye(cxx.shape[0])", "cxx",
     [lambda: affine_pins.test_ridge_normal_equations_two_pass(0.05)]),
    ("affine pooled fit uses one head", "xs = [x.reshape(n * H, d)]\n        ys = [y.reshape(n * H, d)]",
     "xs = [x[:, 0]]\n        ys = [y[:, 0]]",
     [affine_pins.test_pooled_equals_lstsq_on_augmented_system]),
    ("coverage without the softmax scale", "logits = (q[rows, h] @ k[:, h].T) * scale",
     "logits = (q[rows, h] @ k[:, h].T)", [coverage_pins.test_brute_force_rows]),
    ("coverage sums the unselected tiles", "kept = np.flatnonzero(sel[pos[int(row_tile[r])]])",
     "kept = np.flatnonzero(~sel[pos[int(row_tile[r])]])", [coverage_pins.test_all_tiles_kept_covers_all_patch_mass]),
    ("coverage counts special keys as selected", "sel_mass[r, a] = p[r, toks].sum()",
     "sel_mass[r, a] = p[r, toks].sum() + p[r, spec].sum()",
     [coverage_pins.test_all_tiles_kept_covers_all_patch_mass]),
    ("allocation takes the largest errors", 'order = np.argsort(errors, kind="stable")',
     'order = np.argsort(-errors, kind="stable")', [affine_pins.test_allocation_takes_the_lowest_errors]),
    ("allocation count truncated", "count = int(np.floor(linear_fraction * L + 0.5))",
     "count = int(linear_fraction * L)", [affine_pins.test_allocation_takes_the_lowest_errors]),
    ("residual drops the cross term", "- 2.0 * np.trace(Ag @ m[\"sxy\"][gi])", "",
     [affine_pins.test_residual_from_moments_equals_direct_error]),
]


@pytest.mark.parametrize("name,old,new,calls", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, old, new, calls, monkeypatch):
    mod = _mutant(old, new)
    assert _fails(calls, mod, monkeypatch), f"no pin caught: {name}"


def test_unmutated_copy_passes_the_same_pins(monkeypatch):
    mod = _mutant("NEAR_TIE_REL_GAP = 1e-5", "NEAR_TIE_REL_GAP = 1e-5")
    calls = [c for m in MUTATIONS for c in m[3]]
    monkeypatch.setattr(pins, "oracle", mod)
    monkeypatch.setattr(affine_pins, "oracle", mod)
    monkeypatch.setattr(coverage_pins, "oracle", mod)
    for c in calls:
        c()
    assert os.path.exists(zo.__file__)

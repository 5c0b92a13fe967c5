"""Planted mistakes: each one-line change to the oracle's source must make a
named pin of test_oracle_pins fail.

The mutated source is compiled into a fresh in-memory module (the oracle on
disk is not touched) and the pin runs against it in place of the oracle. The
list covers every function of the oracle: the momentum forms, the Nesterov
look-ahead, the normalisation, the Newton-Schulz loop, the shape scale, the
decoupled and cautious updates, the ANVIL wiring, the EMA, the weighted
average, the readout blend, the bf16 rounding, the storage rounding and the
flop count. Rewrites that compute the same values (for example returning
X.T exactly when the input was tall) are not mistakes and are left out.
"""
import inspect
import types

import numpy as np
import pytest

import oracle.muon_oracle as om
import test_oracle_pins as pins

SRC = inspect.getsource(om)

# (what goes wrong, text in the oracle, replacement, pin, pin arguments)
MUTANTS = [
    ("moving average: betas swapped", "return mu * M + (1.0 - mu) * G", "return (1.0 - mu) * M + mu * G",
     "test_anvil_momenta_and_ema_unroll", {}),
    ("moving average: (1 - mu) dropped", "return mu * M + (1.0 - mu) * G", "return mu * M + G",
     "test_momentum_three_step_unroll", {}),
    ("SGD form: (1 - mu) added", "return mu * M + G", "return mu * M + (1.0 - mu) * G",
     "test_sgd_form_three_step_unroll_and_step", {}),
    ("SGD Nesterov: mu on G", "return G + mu * M_new", "return M_new + mu * G",
     "test_sgd_form_three_step_unroll_and_step", {}),
    ("Nesterov: weights swapped", "return (1.0 - mu) * G + mu * M_new", "return mu * G + (1.0 - mu) * M_new",
     "test_momentum_three_step_unroll", {}),
    ("Nesterov: flag ignored", "    if nesterov:\n        return (1.0 - mu) * G + mu * M_new",
     "    if True:\n        return (1.0 - mu) * G + mu * M_new", "test_momentum_three_step_unroll", {}),
    ("Nesterov: U = G", "return (1.0 - mu) * G + mu * M_new", "return G",
     "test_momentum_three_step_unroll", {}),
    ("normalise by the spectral norm", 'np.linalg.norm(U, "fro") + eps', "np.linalg.norm(U, 2) + eps",
     "test_svd_closed_form", dict(shape=(5, 9), cname="cubic5")),
    ("normalise without eps", 'np.linalg.norm(U, "fro") + eps', 'np.linalg.norm(U, "fro")',
     "test_rank_one_update_closed_form", dict(shape=(3, 12))),
    ("normalise by the squared norm", 'np.linalg.norm(U, "fro") + eps', 'np.linalg.norm(U, "fro") ** 2 + eps',
     "test_rank_one_update_closed_form", dict(shape=(3, 12))),
    ("update X B instead of B X on square matrices", "X = a * X + B @ X",
     "X = a * X + (B @ X.T).T if X.shape[0] == X.shape[1] else a * X + B @ X",
     "test_svd_closed_form", dict(shape=(16, 16), cname="quintic5")),
    ("c A instead of c A^2", "B = b * A + c * (A @ A)", "B = b * A + c * A",
     "test_exact_rational_orbit", {}),
    ("b and c swapped", "B = b * A + c * (A @ A)", "B = c * A + b * (A @ A)",
     "test_svd_closed_form", dict(shape=(9, 5), cname="quintic5")),
    ("a dropped", "X = a * X + B @ X", "X = X + B @ X",
     "test_cubic_converges_to_polar_factor", dict(shape=(2, 2))),
    ("Gram of the first iterate every step", "        A = X @ X.T\n", "        A = X0 @ X0.T\n",
     "test_cubic_converges_to_polar_factor", dict(shape=(2, 2))),
    ("last coefficients for every step", "    for a, b, c in coeffs:\n        A = X @ X.T",
     "    for a, b, c in [coeffs[-1]] * len(coeffs):\n        A = X @ X.T",
     "test_svd_closed_form", dict(shape=(5, 9), cname="schedule")),
    ("shape scale inverted", "max(1.0, rows / cols)", "max(1.0, cols / rows)",
     "test_rank_one_update_closed_form", dict(shape=(3, 12))),
    ("shape scale without the square root", "math.sqrt(max(1.0, rows / cols))", "max(1.0, rows / cols)",
     "test_rank_one_update_closed_form", dict(shape=(12, 3))),
    ("shape scale with min", "max(1.0, rows / cols)", "min(1.0, rows / cols)",
     "test_rank_one_update_closed_form", dict(shape=(3, 12))),
    ("decay without lr", "theta * (1.0 - lr * wd) - lr * scale * O", "theta * (1.0 - wd) - lr * scale * O",
     "test_rank_one_update_closed_form", dict(shape=(8, 8))),
    ("update without the shape scale", "theta * (1.0 - lr * wd) - lr * scale * O",
     "theta * (1.0 - lr * wd) - lr * O", "test_rank_one_update_closed_form", dict(shape=(12, 3))),
    ("update with the wrong sign", "theta * (1.0 - lr * wd) - lr * scale * O",
     "theta * (1.0 - lr * wd) + lr * scale * O", "test_rank_one_update_closed_form", dict(shape=(8, 8))),
    ("decay applied after the update", "theta * (1.0 - lr * wd) - lr * scale * O",
     "(theta - lr * scale * O) * (1.0 - lr * wd)", "test_rank_one_update_closed_form", dict(shape=(8, 8))),
    ("mask inverted", "(O * M_slow > 0.0)", "(O * M_slow < 0.0)", "test_cautious_mask_closed_form", {}),
    ("mask where the product is zero", "(O * M_slow > 0.0)", "(O * M_slow >= 0.0)",
     "test_anvil_tall_rank_one_with_zero_rows_closed_form", {}),
    ("cautious decay without the mask", "lr * wd * mask * theta", "lr * wd * theta",
     "test_cautious_mask_closed_form", {}),
    ("mask on the update instead of the decay",
     "return theta - lr * wd * mask * theta - lr * scale * O",
     "return theta - lr * wd * theta - lr * scale * mask * O", "test_cautious_mask_closed_form", {}),
    ("cautious update without the shape scale", "- lr * wd * mask * theta - lr * scale * O",
     "- lr * wd * mask * theta - lr * O", "test_anvil_tall_rank_one_with_zero_rows_closed_form", {}),
    ("ANVIL orthogonalises the slow momentum", "O = orthogonalize(Mf, hp", "O = orthogonalize(Ms, hp",
     "test_anvil_step_wiring_three_steps_closed_form", {}),
    ("ANVIL mask from the fast momentum", "mask = cautious_mask(O, Ms)", "mask = cautious_mask(O, Mf)",
     "test_anvil_step_wiring_three_steps_closed_form", {}),
    ("ANVIL mask from the gradient", "mask = cautious_mask(O, Ms)", "mask = cautious_mask(O, G)",
     "test_cautious_mask_closed_form", {}),
    ("ANVIL betas swapped",
     'Mf = momentum_update(as_f64(M_fast), G, hp["beta_fast"])\n    Ms = momentum_update(as_f64(M_slow), G, hp["beta_slow"])',
     'Mf = momentum_update(as_f64(M_fast), G, hp["beta_slow"])\n    Ms = momentum_update(as_f64(M_slow), G, hp["beta_fast"])',
     "test_anvil_step_wiring_three_steps_closed_form", {}),
    ("ANVIL decays every element", "theta_new = cautious_update(theta, O, mask,",
     "theta_new = cautious_update(theta, O, np.ones_like(mask),", "test_cautious_mask_closed_form", {}),
    ("EMA weights swapped", "return beta * as_f64(ema) + (1.0 - beta) * as_f64(theta)",
     "return (1.0 - beta) * as_f64(ema) + beta * as_f64(theta)", "test_anvil_momenta_and_ema_unroll", {}),
    ("weighted average divided by the count", "    return acc / sum(w)", "    return acc / len(w)",
     "test_weighted_average_three_checkpoints_by_hand", {}),
    ("running-average beta w/W instead of 1 - w/W", "out.append(1.0 - float(wn) / W if W > 0.0 else 0.0)",
     "out.append(float(wn) / W if W > 0.0 else 0.0)", "test_weighted_average_running_form_exact_rationals", {}),
    ("readout weights swapped", "return w_final * as_f64(theta) + (1.0 - w_final) * as_f64(ema)",
     "return (1.0 - w_final) * as_f64(theta) + w_final * as_f64(ema)", "test_page_constants", {}),
    ("readout default 0.65", "w_final: float = 0.35", "w_final: float = 0.65", "test_page_constants", {}),
    ("bf16 by truncation", "np.rint(m * 256.0)", "np.trunc(m * 256.0)", "test_round_to_bf16_matches_torch", {}),
    ("bf16 with 7 significant bits", "np.ldexp(np.rint(m * 256.0), e - 8)", "np.ldexp(np.rint(m * 128.0), e - 7)",
     "test_round_to_bf16_matches_torch", {}),
    ("bf16 ties away from zero", "np.rint(m * 256.0)", "np.sign(m) * np.floor(np.abs(m * 256.0) + 0.5)",
     "test_round_to_bf16_matches_torch", {}),
    ("f32 storage not rounded",
     "return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)",
     "return np.asarray(x, dtype=np.float64)", "test_sgd_form_three_step_unroll_and_step", {}),
    ("flop count: full Gram", "r * (r + 1) * c + r * r * (r + 1) + 2.0 * r * r * c",
     "r * r * c + r * r * (r + 1) + 2.0 * r * r * c", "test_flop_count_by_counting_operations", dict(shape=(3, 5))),
    ("flop count: dense products", "r * (r + 1) * c + r * r * (r + 1) + 2.0 * r * r * c",
     "2.0 * r * r * c + 2.0 * r * r * r + 2.0 * r * r * c",
     "test_flop_count_matches_dense_count_minus_symmetry", {}),
    ("muon_step: shape scale of the transpose", "shape_scale(rows, cols))\n    return round_to_storage(theta_new, param_dtype), M_new, O",
     "shape_scale(cols, rows))\n    return round_to_storage(theta_new, param_dtype), M_new, O",
     "test_rank_one_update_closed_form", dict(shape=(3, 12))),
    ("muon_step: SGD form ignores Nesterov", 'U = nesterov_lookahead_sgd(M_new, G, hp["mu"], bool(hp["nesterov"]))',
     "U = M_new", "test_sgd_form_step_on_diagonal_matrices_closed_form", dict(nesterov=1)),
    ("muon_step: parameters not rounded to storage",
     "    return round_to_storage(theta_new, param_dtype), M_new, O", "    return theta_new, M_new, O",
     "test_sgd_form_three_step_unroll_and_step", {}),
]


def _module(src):
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src, "oracle_mutant", "exec"), mod.__dict__)
    return mod


def _run_pin(monkeypatch, mod, pin, kw):
    """True if the pin passes with `mod` in place of the oracle."""
    monkeypatch.setattr(pins, "oracle", mod)
    try:
        with np.errstate(all="ignore"):
            getattr(pins, pin)(**kw)
        return True
    except Exception:
        return False


@pytest.mark.parametrize("pin,kw", sorted({(m[3], tuple(sorted(m[4].items()))) for m in MUTANTS}))
def test_every_pin_used_passes_on_the_unchanged_source(monkeypatch, pin, kw):
    assert _run_pin(monkeypatch, _module(SRC), pin, dict(kw))


@pytest.mark.parametrize("what,old,new,pin,kw", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_its_pin(monkeypatch, what, old, new, pin, kw):
    assert SRC.count(old) == 1, "the mutated text must occur exactly once"
    assert not _run_pin(monkeypatch, _module(SRC.replace(old, new)), pin, kw), what

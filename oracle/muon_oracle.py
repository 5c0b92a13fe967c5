"""Double-precision CPU oracle for the Muon / ANVIL optimizer step.

TEST INFRASTRUCTURE ONLY. The tests, the smoke check in ``__graft_entry__`` and
the CPU-baseline leg of ``bench.py`` are the only callers allowed. The product
path (the CUDA library and its Python binding) never imports or calls this
module, and this module imports nothing from the product path.

Everything runs in float64 on dense matrices, one matrix at a time, in the order
the method states its steps. ``numpy.matmul`` and ``numpy.linalg.norm`` are the
only library primitives. There is no symmetric shortcut, no blocking and no
fusion, so each function can be checked against its source by eye.

Sources (pages as titled; sections in brackets):
  [P1] "きみはNanoGPT speedrunを知っているか？" (prednext.com), section "Muonとは":
       Muon keeps a moving average of the gradient (momentum), approximately
       orthogonalises it with a Newton-Schulz iteration and updates the
       parameters with the result; it applies only to matrix parameters.
  [P4] neo-ai.one article on Keller Jordan, section "Muonが登場": the update
       matrix from SGD-momentum is orthogonalised by Newton-Schulz iteration
       toward a semi-orthogonal matrix; the iteration runs stably in bf16.
  [P3] "Training NanoGPT in 39.9 Seconds", section "ANVIL II와 가중치 평균":
       ANVIL keeps a fast and a slow momentum, applies a polynomial map six times
       to the update to flatten its singular values, and chooses the elements
       that receive cautious weight decay by agreement with the slow momentum;
       end-of-training averaging uses the EMA
       theta_bar_t = beta * theta_bar_{t-1} + (1 - beta) * theta_t  (0 <= beta < 1),
       and the readout mixes 35 % final weights with 65 % of the average.
  [P2] "qlabs-eng/slowrun", section "仕組み": the baseline trains with Muon and
       a very high weight decay (1.6).

The pages give the Newton-Schulz step only by name. The odd polynomial step
X <- a X + (b A + c A^2) X with A = X X^T, Frobenius normalisation beforehand,
the transpose rule for tall matrices, the shape scale max(1, R/C)^(1/2) and
decoupled weight decay are the method statement this oracle encodes. Where the
pages leave a step open the plainest reading is taken; each reading is named at
the function that takes it:
  R1  momentum is the moving average  M <- mu M + (1 - mu) G ("Muonとは").
  R2  Nesterov look-ahead  U = (1 - mu) G + mu M  with the updated M.
  R3  X0 = U / (||U||_F + eps).
  R4  tall matrices (R > C) are iterated on the transpose and transposed back.
  R5  decoupled decay multiplies lr: theta <- theta (1 - lr wd) - lr s O.
  R6  ANVIL orthogonalises the fast momentum; the slow one only picks the mask.
  R7  the cautious mask is O * M_slow > 0 (strict: zeros are not decayed).
  R8  the EMA starts at the parameters' value when averaging starts.
  R16 a parameter write rounds to the parameter's storage type to nearest even.

Parity status: every function here is pinned by tests (SVD closed form, cubic
convergence to the polar factor, hand-unrolled recurrences, invariants, exact
rational orbits and the page constants); none is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Sequence

import numpy as np

__all__ = [
    "as_f64",
    "round_to_bf16",
    "round_to_storage",
    "momentum_update",
    "momentum_update_sgd",
    "nesterov_lookahead",
    "nesterov_lookahead_sgd",
    "frobenius_normalize",
    "newton_schulz",
    "orthogonalize",
    "shape_scale",
    "decoupled_update",
    "cautious_mask",
    "cautious_update",
    "muon_step",
    "anvil_step",
    "ema_update",
    "weighted_average",
    "weighted_average_betas",
    "readout_blend",
    "ns_flops_algorithmic",
]


# --------------------------------------------------------------------------
# storage types
# --------------------------------------------------------------------------
def as_f64(x) -> np.ndarray:
    """Exact upcast of a float32 / bfloat16 / float64 host array to float64.

    Accepts numpy arrays or CPU torch tensors (converted through float32, which
    represents every bfloat16 value exactly).
    """
    if hasattr(x, "detach"):  # torch tensor, without importing torch here
        x = x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float64)


def round_to_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even (R16).

    bfloat16 keeps 8 significant bits and float32's exponent range. The value
    is split as m * 2**e with 0.5 <= |m| < 1; m * 2**8 is rounded to the
    nearest integer with ties to even (numpy.rint), then scaled back. Values
    below float32's normal range or above its maximum do not occur in this
    method and are not treated specially.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def round_to_storage(x, dtype: str) -> np.ndarray:
    """Round to the parameter storage type: 'bf16' (RNE) or 'f32' (RNE)."""
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(f"unknown storage type {dtype!r}")


# --------------------------------------------------------------------------
# Muon, step by step
# --------------------------------------------------------------------------
def momentum_update(M: np.ndarray, G: np.ndarray, mu: float) -> np.ndarray:
    """Moving average of the gradient, M <- mu M + (1 - mu) G.

    [P1] "Muonとは" calls the momentum a moving average of the gradient (R1).
    """
    return mu * M + (1.0 - mu) * G


def momentum_update_sgd(M: np.ndarray, G: np.ndarray, mu: float) -> np.ndarray:
    """SGD-form momentum M <- mu M + G (the "SGD-momentum" of "Muonが登場"),
    the alternative to R1 that a flag selects."""
    return mu * M + G


def nesterov_lookahead_sgd(M_new: np.ndarray, G: np.ndarray, mu: float,
                           nesterov: bool) -> np.ndarray:
    """U = G + mu M for the SGD form with Nesterov, else U = M."""
    if nesterov:
        return G + mu * M_new
    return M_new


def nesterov_lookahead(M_new: np.ndarray, G: np.ndarray, mu: float,
                       nesterov: bool) -> np.ndarray:
    """The matrix that gets orthogonalised: U = (1 - mu) G + mu M if Nesterov,
    else U = M (R2; the Nesterov option belongs to the method statement)."""
    if nesterov:
        return (1.0 - mu) * G + mu * M_new
    return M_new


def frobenius_normalize(U: np.ndarray, eps: float) -> np.ndarray:
    """X0 = U / (||U||_F + eps) (R3). Frobenius >= spectral norm, so every
    singular value of X0 is at most 1."""
    return U / (np.linalg.norm(U, "fro") + eps)


def newton_schulz(X0: np.ndarray, coeffs: Sequence[Sequence[float]]) -> np.ndarray:
    """Iterate X <- a X + (b A + c A @ A) X with A = X X^T, once per (a, b, c).

    [P1] "Muonとは" / [P4] "Muonが登場": the momentum is orthogonalised
    approximately by Newton-Schulz iteration. X0 must have rows <= cols, so A
    is the smaller (rows x rows) Gram matrix. Dense products throughout.
    """
    X = np.array(X0, dtype=np.float64, copy=True)
    if X.shape[0] > X.shape[1]:
        raise ValueError("newton_schulz expects rows <= cols; use orthogonalize")
    for a, b, c in coeffs:
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X


def orthogonalize(U: np.ndarray, coeffs: Sequence[Sequence[float]],
                  eps: float) -> np.ndarray:
    """O = NS(U / (||U||_F + eps)), iterating on U^T when U is tall (R4)."""
    U = as_f64(U)
    tall = U.shape[0] > U.shape[1]
    X = U.T if tall else U
    X = newton_schulz(frobenius_normalize(X, eps), coeffs)
    return X.T if tall else X


def shape_scale(rows: int, cols: int) -> float:
    """s = max(1, rows / cols) ** 0.5."""
    return math.sqrt(max(1.0, rows / cols))


def decoupled_update(theta: np.ndarray, O: np.ndarray, lr: float, wd: float,
                     scale: float) -> np.ndarray:
    """theta <- theta (1 - lr wd) - lr s O (R5). [P2] "仕組み" names the very
    high weight decay 1.6, which only makes sense multiplied by lr."""
    return theta * (1.0 - lr * wd) - lr * scale * O


def cautious_mask(O: np.ndarray, M_slow: np.ndarray) -> np.ndarray:
    """1.0 where the update agrees in sign with the slow momentum, else 0.0.

    [P3] "ANVIL II와 가중치 평균": the elements that get cautious weight decay
    are chosen by agreement with the slow momentum (R7: O * M_slow > 0).
    """
    return (O * M_slow > 0.0).astype(np.float64)


def cautious_update(theta: np.ndarray, O: np.ndarray, mask: np.ndarray,
                    lr: float, wd: float, scale: float) -> np.ndarray:
    """theta <- theta - lr wd mask * theta - lr s O."""
    return theta - lr * wd * mask * theta - lr * scale * O


def muon_step(theta, G, M, hp: dict, param_dtype: str):
    """One Muon step on one matrix.

    hp keys: lr, mu, weight_decay, nesterov, coeffs (list of (a, b, c)), eps,
    and optionally sgd_momentum (SGD-form buffer instead of the moving average).
    Returns (theta_new rounded to param_dtype, M_new, O).
    """
    theta = as_f64(theta)
    G = as_f64(G)
    M = as_f64(M)
    rows, cols = theta.shape
    if hp.get("sgd_momentum"):
        M_new = momentum_update_sgd(M, G, hp["mu"])
        U = nesterov_lookahead_sgd(M_new, G, hp["mu"], bool(hp["nesterov"]))
    else:
        M_new = momentum_update(M, G, hp["mu"])
        U = nesterov_lookahead(M_new, G, hp["mu"], bool(hp["nesterov"]))
    O = orthogonalize(U, hp["coeffs"], hp["eps"])
    theta_new = decoupled_update(theta, O, hp["lr"], hp["weight_decay"],
                                 shape_scale(rows, cols))
    return round_to_storage(theta_new, param_dtype), M_new, O


def anvil_step(theta, G, M_fast, M_slow, hp: dict, param_dtype: str):
    """One ANVIL-style step on one matrix ([P3] "ANVIL II와 가중치 평균").

    Both momenta are moving averages (beta_fast, beta_slow). The fast one is
    orthogonalised (R6) with the given polynomial list (six applications in the
    pages' recipe), and the decay is masked by sign agreement with the slow one.
    Returns (theta_new rounded, M_fast_new, M_slow_new, O, mask).
    """
    theta = as_f64(theta)
    G = as_f64(G)
    rows, cols = theta.shape
    Mf = momentum_update(as_f64(M_fast), G, hp["beta_fast"])
    Ms = momentum_update(as_f64(M_slow), G, hp["beta_slow"])
    O = orthogonalize(Mf, hp["coeffs"], hp["eps"])
    mask = cautious_mask(O, Ms)
    theta_new = cautious_update(theta, O, mask, hp["lr"], hp["weight_decay"],
                                shape_scale(rows, cols))
    return round_to_storage(theta_new, param_dtype), Mf, Ms, O, mask


def ema_update(ema: np.ndarray, theta: np.ndarray, beta: float) -> np.ndarray:
    """theta_bar <- beta theta_bar + (1 - beta) theta
    ([P3] "ANVIL II와 가중치 평균", the averaging equation)."""
    return beta * as_f64(ema) + (1.0 - beta) * as_f64(theta)


def weighted_average(thetas: Sequence, weights: Sequence[float]) -> np.ndarray:
    """theta_bar = sum_i w_i theta_i / sum_i w_i over checkpoints theta_i.

    "qlabs-eng/slowrun", leaderboard table: weighted checkpoint averaging. The
    page gives no weights, so they are the caller's (w_i >= 0, sum > 0). The
    EMA of "ANVIL II와 가중치 평균" is the special case w_0 = beta^n,
    w_i = (1 - beta) beta^(n - i).
    """
    w = [float(x) for x in weights]
    if len(w) != len(thetas) or not w or min(w) < 0.0 or sum(w) <= 0.0:
        raise ValueError("need one non-negative weight per checkpoint, not all zero")
    acc = np.zeros_like(as_f64(thetas[0]))
    for wi, th in zip(w, thetas):
        acc = acc + wi * as_f64(th)
    return acc / sum(w)


def weighted_average_betas(weights: Sequence[float]) -> list:
    """The decay of each checkpoint that makes the EMA recurrence
    theta_bar <- beta_n theta_bar + (1 - beta_n) theta_n produce the running
    weighted average: beta_n = 1 - w_n / W_n with W_n = w_1 + ... + w_n
    (beta_1 = 0, so the average starts at the first checkpoint). Checkpoints
    before the first positive weight get beta = 1 - 0 / 0, taken as 0 here
    (they are overwritten by the first weighted one)."""
    out, W = [], 0.0
    for wn in weights:
        W += float(wn)
        out.append(1.0 - float(wn) / W if W > 0.0 else 0.0)
    return out


def readout_blend(theta: np.ndarray, ema: np.ndarray, w_final: float = 0.35) -> np.ndarray:
    """out = w_final theta + (1 - w_final) theta_bar; the pages' readout uses
    35 % final weights and 65 % average ([P3] "ANVIL II와 가중치 평균")."""
    return w_final * as_f64(theta) + (1.0 - w_final) * as_f64(ema)


# --------------------------------------------------------------------------
# bookkeeping used by the benchmark's roofline line
# --------------------------------------------------------------------------
def ns_flops_algorithmic(rows: int, cols: int, steps: int) -> float:
    """Algorithmic flops of `steps` iterations on one rows x cols matrix with
    a symmetric Gram and square: r(r+1)c + r^2(r+1) + 2 r^2 c per iteration,
    r = min, c = max."""
    r, c = min(rows, cols), max(rows, cols)
    return float(steps) * (r * (r + 1) * c + r * r * (r + 1) + 2.0 * r * r * c)


"""One optimizer step of a bank, checked against the CPU oracle (test helper).

Given a bank's state before and after one step of the CUDA path, and the
gradient it was given, these checks recompute the step with the oracle:
  * momentum (both momenta for ANVIL) on every element, within 1e-5;
  * on the picked matrices, the parameter step theta_new - theta_old against
    the oracle's (relative Frobenius 2e-2 after one storage ulp per element);
  * with fp32 parameters, the orthogonalised update O recovered from the step
    (the decay term is known, so O = (theta_old (1 - lr wd) - theta_new) /
    (lr s)), against the oracle's O: relative Frobenius 2e-2 and every
    singular value within 0.05.
"""
import numpy as np

import oracle
from _parity import TOL_BUFFER, buffer_ok, delta_ok, rel_fro, sv_maxdiff, update_tols


def f64(t):
    return oracle.as_f64(t.detach().cpu())


def check_muon_step(th0, th1, G, M0, M1, hp, picks, param_dtype):
    """Muon (moving-average or SGD-form momentum, Nesterov or not)."""
    G, M0, M1, th0, th1 = f64(G), f64(M0), f64(M1), f64(th0), f64(th1)
    sgd = bool(hp.get("sgd_momentum"))
    upd = oracle.momentum_update_sgd if sgd else oracle.momentum_update
    look = oracle.nesterov_lookahead_sgd if sgd else oracle.nesterov_lookahead
    Mref = upd(M0, G, hp["mu"])
    ok, r = buffer_ok(M1, Mref, TOL_BUFFER)
    assert ok, ("momentum", r)
    R, C = th0.shape[1:]
    s = oracle.shape_scale(R, C)
    tol_o, tol_sv = update_tols(R, C)
    for i in picks:
        U = look(Mref[i], G[i], hp["mu"], bool(hp["nesterov"]))
        O = oracle.orthogonalize(U, hp["coeffs"], hp["eps"])
        dref = oracle.decoupled_update(th0[i], O, hp["lr"], hp["weight_decay"], s) - th0[i]
        ok, r = delta_ok(th0[i], th1[i], dref, param_dtype, tol_o)
        assert ok, ("delta", i, r)
        if param_dtype == "f32":
            Og = (th0[i] * (1.0 - hp["lr"] * hp["weight_decay"]) - th1[i]) / (hp["lr"] * s)
            assert rel_fro(Og, O) <= tol_o, ("O", i, rel_fro(Og, O))
            assert sv_maxdiff(Og, O) <= tol_sv, ("singular values", i, sv_maxdiff(Og, O))


def check_anvil_step(th0, th1, G, Mf0, Mf1, Ms0, Ms1, hp, picks, param_dtype):
    """ANVIL: both momenta, cautious decay; O is recovered when wd = 0."""
    G, th0, th1 = f64(G), f64(th0), f64(th1)
    Mf = oracle.momentum_update(f64(Mf0), G, hp["beta_fast"])
    Ms = oracle.momentum_update(f64(Ms0), G, hp["beta_slow"])
    ok, r = buffer_ok(f64(Mf1), Mf)
    assert ok, ("fast momentum", r)
    ok, r = buffer_ok(f64(Ms1), Ms)
    assert ok, ("slow momentum", r)
    R, C = th0.shape[1:]
    s = oracle.shape_scale(R, C)
    tol_o, tol_sv = update_tols(R, C)
    for i in picks:
        O = oracle.orthogonalize(Mf[i], hp["coeffs"], hp["eps"])
        mask = oracle.cautious_mask(O, Ms[i])
        dref = oracle.cautious_update(th0[i], O, mask, hp["lr"], hp["weight_decay"], s) - th0[i]
        ok, r = delta_ok(th0[i], th1[i], dref, param_dtype, tol_o)
        assert ok, ("anvil delta", i, r)
        if param_dtype == "f32" and hp["weight_decay"] == 0.0:
            Og = (th0[i] - th1[i]) / (hp["lr"] * s)
            assert rel_fro(Og, O) <= tol_o, ("O", i, rel_fro(Og, O))
            assert sv_maxdiff(Og, O) <= tol_sv


def hp_dict(hp):
    """An Hparams object as the oracle's dict (plain numbers)."""
    return dict(lr=hp.lr, mu=hp.mu, weight_decay=hp.weight_decay, eps=hp.eps,
                nesterov=1 if hp.nesterov else 0, coeffs=[tuple(c) for c in hp.coeffs],
                ema_beta=hp.ema_beta, beta_fast=hp.beta_fast, beta_slow=hp.beta_slow,
                sgd_momentum=1 if hp.sgd_momentum else 0)

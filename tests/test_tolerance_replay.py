"""Where the GPU parity tolerances come from (CPU only).

A float64 replay of the rounding that the Newton-Schulz kernel applies (a
model written for this test; the oracle knows nothing of it):
  - every GEMM operand is bf16: the iterate's high part X_hi, A and B;
  - products accumulate in fp32 (modelled as a float64 product rounded to
    fp32); A and B are stored as bf16;
  - the iterate is carried as a bf16 pair hi + lo and the a*X term uses both;
  - step 0 runs on the stored U and folds s = 1/(||U|| + eps) into the
    epilogues: A = s^2 U_hi U_hi^T, X_1 = s (a U + B U_hi).
Tall matrices are replayed on the transpose. The replay's distance to the
oracle on the parity tests' own inputs must sit inside the tolerances those
tests use, and dropping the low half of the iterate must break them on the
spiked GPT gradients, which is why the kernel carries it.
"""
import numpy as np
import pytest
import torch

import muon_inputs as mi
import oracle
from _parity import TOL_SV, TOL_UPDATE, rel_fro, sv_maxdiff, update_tols


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _mm(a, b):
    return _f32(a @ b)


def replay_orthogonalize(u, coeffs, eps=1e-7, keep_lo=True, lo_steps=None):
    """The kernel's arithmetic for one matrix (rows <= cols after transposing).
    lo_steps (not the kernel: a variant to test against) carries the low half
    only into the a*X term of the first lo_steps steps."""
    tall = u.shape[0] > u.shape[1]
    u = _f32(u.T if tall else u)
    s = 1.0 / (np.sqrt(np.sum(u * u)) + eps)
    hi = _bf16(u)
    lo = _bf16(u - hi) if keep_lo else np.zeros_like(u)
    for k, (a, b, c) in enumerate(coeffs):
        scale = s if k == 0 else 1.0
        A = _bf16(_f32(scale * scale * _mm(hi, hi.T)))
        B = _bf16(_f32(b * A + c * _mm(A, A)))
        use_lo = lo if lo_steps is None or k < lo_steps else 0.0
        x = _f32(a * scale * (hi + use_lo) + scale * _mm(B, hi))
        hi = _bf16(x)
        lo = _bf16(x - hi) if keep_lo else np.zeros_like(x)
    out = hi + lo
    return out.T if tall else out


Q5 = [mi.QUINTIC] * 5
Q6 = [mi.QUINTIC] * 6
CASES = [  # (count, rows, cols, coefficient list), the GPU orthogonalisation test's inputs
    (2, 7, 13, Q6), (2, 13, 7, Q6), (2, 7, 13, Q5), (1, 129, 257, Q5), (1, 257, 129, Q6),
    (1, 256, 512, Q5), (2, 384, 640, Q6), (1, 256, 512, [mi.CUBIC] * 5),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c}x{r}x{k}-{len(co)}" for c, r, k, co in CASES])
def test_replayed_kernel_rounding_fits_the_parity_tolerances(case):
    cnt, R, C, coeffs = case
    g = mi.gaussian(cnt * R, C, seed=R * 1000 + C, sigma=1.0).reshape(cnt, R, C).to(torch.bfloat16)
    tol, sv_tol = update_tols(R, C)
    if coeffs[0] == mi.CUBIC:
        tol = 5e-3  # the GPU test's cubic tolerance
    for i in range(cnt):
        u = g[i].double().numpy()
        ref = oracle.orthogonalize(u, coeffs, 1e-7)
        got = replay_orthogonalize(u, coeffs)
        assert rel_fro(got, ref) <= tol, (i, rel_fro(got, ref), tol)
        assert sv_maxdiff(got, ref) <= sv_tol, (i, sv_maxdiff(got, ref), sv_tol)


def test_the_low_half_of_the_iterate_is_needed_on_spiked_gradients():
    """GPT-bank-like gradient (N(0, 1e-3^2) plus a rank-4 spike at 10x RMS):
    with the hi + lo iterate the replay is far inside 2e-2; with a bf16-only
    iterate it is not."""
    u = mi.spiked_gaussian(768, 768, 1, 1e-3, 4, 10.0).double().numpy()
    ref = oracle.orthogonalize(u, Q5, 1e-7)
    with_lo = rel_fro(replay_orthogonalize(u, Q5), ref)
    without = rel_fro(replay_orthogonalize(u, Q5, keep_lo=False), ref)
    assert with_lo < 0.25 * TOL_UPDATE, with_lo
    assert without > TOL_UPDATE, without
    assert sv_maxdiff(replay_orthogonalize(u, Q5), ref) < TOL_SV


def test_the_low_half_is_needed_in_every_step_on_low_rank_gradients():
    """A rank-64 gradient (x^T dy over 64 rows, as one batch of 64 gives). Its
    null space has singular value 0: there B X vanishes and only the a X term
    acts, multiplying the iterate's rounding noise by a (about 3.4) every
    step. With the low half in every step (the kernel) the replay stays far
    inside the tolerance; carried only into the first two steps, the noise
    grows past it by step 5 (the GPU kernel built that way measured 8.5e-2
    and 0.24 on such gradients, as this replay predicts)."""
    g = torch.Generator().manual_seed(11)
    x = torch.randn(64, 768, generator=g, dtype=torch.float64)
    dy = torch.randn(64, 768, generator=g, dtype=torch.float64)
    u = (x.T @ dy).to(torch.bfloat16).double().numpy()
    for coeffs in (Q5, Q6):
        ref = oracle.orthogonalize(u, coeffs, 1e-7)
        assert rel_fro(replay_orthogonalize(u, coeffs), ref) < 0.5 * TOL_UPDATE
        assert rel_fro(replay_orthogonalize(u, coeffs, lo_steps=2), ref) > 2 * TOL_UPDATE

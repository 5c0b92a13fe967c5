"""Comparison helpers shared by the GPU parity tests (no method arithmetic)."""
import numpy as np

# Tolerances of the method statement.
TOL_BUFFER = 1e-5      # fp32 momentum / EMA buffers, relative
TOL_UPDATE = 2e-2      # orthogonalised update, relative Frobenius
TOL_SV = 0.05          # every output singular value, absolute


def update_tols(rows, cols):
    """(relative Frobenius, singular-value) tolerances of the orthogonalised
    update. With fewer than 32 singular values one bf16-sensitive value
    dominates: replaying the kernel's own bf16 rounding scheme in float64 on
    the CPU gives up to 3.3e-2 / 0.057 on 7 x 13 and 2.1e-2 on 8 x 1, so tiny
    matrices get 4e-2 / 0.08."""
    if min(rows, cols) < 32:
        return 4e-2, 0.08
    return TOL_UPDATE, TOL_SV


def rel_fro(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def buffer_ok(got, ref, tol=TOL_BUFFER):
    """Relative Frobenius within tol and |d| <= tol (|ref| + rms(ref)) per element."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    elem = np.abs(got - ref) <= tol * (np.abs(ref) + rms) + 1e-30
    return rel_fro(got, ref) <= tol and bool(np.all(elem)), rel_fro(got, ref)


def sv_maxdiff(got, ref):
    s1 = np.linalg.svd(np.asarray(got, dtype=np.float64), compute_uv=False)
    s2 = np.linalg.svd(np.asarray(ref, dtype=np.float64), compute_uv=False)
    return float(np.max(np.abs(s1 - s2)))


def bf16_ulp(x):
    """Spacing of bfloat16 values at |x| (8 significant bits)."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def delta_ok(theta_old, theta_new_gpu, delta_ref, dtype, tol=TOL_UPDATE):
    """Parameter step parity: the GPU's theta_new - theta_old against the
    oracle's unrounded step, relative Frobenius <= tol after allowing one
    storage ulp of theta_new per element (the GPU rounds the stored value)."""
    d_gpu = np.asarray(theta_new_gpu, np.float64) - np.asarray(theta_old, np.float64)
    err = np.abs(d_gpu - delta_ref)
    ulp = bf16_ulp(theta_new_gpu) if dtype == "bf16" else np.abs(theta_new_gpu) * 2.0 ** -23
    excess = np.maximum(err - ulp, 0.0)
    r = float(np.linalg.norm(excess) / max(np.linalg.norm(delta_ref), 1e-300))
    return r <= tol, r

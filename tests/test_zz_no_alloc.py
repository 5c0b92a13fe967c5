"""muon_orthogonalize_static: the orthogonalisation for callers that cannot
allocate device memory (for example a plug-in whose host application owns all
device allocations, or a loop where a cudaMalloc that may synchronise the
device is not allowed). Its scratch is the library's own fixed device array.

The test calls the entry point through the C ABI (ctypes) twice in a row, with
different inputs, and compares each result with muon_orthogonalize run on a
caller-owned workspace. Both run the same deterministic kernels on the same
inputs, so the results must be identical bit for bit (any difference means
the fixed scratch was laid out or cleared wrongly); each result is also
within the update tolerance of the CPU oracle. This file is collected last so
that a run stopping at the first failure has run every other test first; it
also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import muon_inputs as mi
import oracle

pytestmark = pytest.mark.gpu

TOL_UPDATE = 2e-2  # orthogonalised update, relative Frobenius (same as the parity tests)


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def test_static_scratch_matches_workspace_entry_point():
    import muon_newton_schulz_05_b200 as mb

    lib = mb.raw_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    hp = mb.Hparams(coeffs=[mi.QUINTIC] * 5, eps=1e-7)
    chp = hp.to_c()
    cases = [(2, 384, 640, 11), (1, 768, 3072, 12)]  # two calls in a row, different shapes
    for cnt, R, C, seed in cases:
        x = mi.spiked_gaussian(cnt * R, C, seed, 1e-3, 4, 10.0).reshape(cnt, R, C)
        x = x.to(torch.bfloat16).to(dev)
        out_static = torch.full((cnt, R, C), float("nan"), device=dev)
        code = lib.muon_orthogonalize_static(x.data_ptr(), mb.BF16, out_static.data_ptr(), mb.F32,
                                             cnt, R, C, ctypes.byref(chp), stream.cuda_stream)
        assert code == 0, mb.status_string(code)
        ws = mb.alloc_workspace([(cnt, R, C)], device=dev)
        out_ws = torch.empty(cnt, R, C, device=dev)
        mb.orthogonalize(x, out_ws, hp, ws)
        torch.cuda.synchronize()
        assert mb.device_status(ws) == 0
        assert torch.isfinite(out_static).all()
        assert torch.equal(out_static, out_ws)
        ref = oracle.orthogonalize(oracle.as_f64(x[0].cpu()), hp.coeffs, hp.eps)
        assert _rel(oracle.as_f64(out_static[0].cpu()), ref) <= TOL_UPDATE


def test_static_scratch_rejects_banks_beyond_its_size():
    import muon_newton_schulz_05_b200 as mb

    lib = mb.raw_library()
    chp = mb.Hparams().to_c()
    fake = 1 << 20  # never dereferenced: the size check comes first
    code = lib.muon_orthogonalize_static(fake, mb.BF16, fake * 64, mb.F32, 1, 2560, 2560,
                                         ctypes.byref(chp), None)
    assert code == 6  # MUON_ERR_WORKSPACE

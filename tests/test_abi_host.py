"""Host-side checks of the C ABI (no GPU needed).

The library loads on a machine without a GPU (the CUDA runtime is linked
statically and only touched after argument validation), so every validation
path and the workspace planner can be exercised here.
"""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import muon_newton_schulz_05_b200 as mb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon_b200.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(mb.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(mb.EXPORTED) == names


def test_version_and_strings():
    assert mb.abi_version() == 2
    for code, name in mb.STATUS_NAMES.items():
        assert mb.status_string(code).startswith(name)
    assert "unknown" in mb.status_string(77)


def test_struct_layout_matches_header():
    """Compile a probe against the header with gcc and compare with ctypes."""
    probe = r'''
#include <stdio.h>
#include <stddef.h>
#include "muon_b200.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu\n", sizeof(muon_bank), offsetof(muon_bank, grad),
         offsetof(muon_bank, ema), sizeof(muon_hparams), offsetof(muon_hparams, coeffs),
         offsetof(muon_hparams, beta_slow), offsetof(muon_hparams, sgd_momentum));
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "p.c")
        exe = os.path.join(d, "p")
        open(c, "w").write(probe)
        subprocess.check_call(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), c, "-o", exe])
        got = [int(x) for x in subprocess.check_output([exe]).split()]
    want = [ctypes.sizeof(mb.CBank), mb.CBank.grad.offset, mb.CBank.ema.offset,
            ctypes.sizeof(mb.CHparams), mb.CHparams.coeffs.offset, mb.CHparams.beta_slow.offset,
            mb.CHparams.sgd_momentum.offset]
    assert got == want


def test_workspace_size_planning():
    s1 = mb.workspace_size([(1, 256, 512)])
    # 3 iterate buffers 256x512 bf16, A and B 256^2 bf16, header and small arrays
    assert s1 >= 3 * 256 * 512 * 2 + 2 * 256 * 256 * 2
    assert mb.workspace_size([(2, 256, 512)]) > s1
    # padding to multiples of 256 in both directions
    assert mb.workspace_size([(1, 7, 13)]) == mb.workspace_size([(1, 256, 256)])
    # tall and wide banks share the Gram size
    assert mb.workspace_size([(3, 768, 3072)]) == mb.workspace_size([(3, 3072, 768)])
    assert mb.workspace_size([(0, 4, 4)]) == 0
    assert mb.workspace_size([(1, 0, 4)]) == 0
    assert mb.workspace_size([]) == 0
    assert mb.workspace_size([(1, 8, 8)] * 9) == 0  # more than MUON_MAX_BANKS


FAKE = 0x10000  # aligned, never dereferenced: validation fails first


def _bank(**kw):
    b = mb.CBank()
    b.count, b.rows, b.cols = kw.get("count", 1), kw.get("rows", 8), kw.get("cols", 8)
    b.param = kw.get("param", FAKE)
    b.param_dtype = kw.get("param_dtype", mb.BF16)
    b.grad = kw.get("grad", FAKE + 0x1000)
    b.grad_dtype = kw.get("grad_dtype", mb.BF16)
    b.momentum = kw.get("momentum", FAKE + 0x2000)
    b.momentum_slow = kw.get("momentum_slow", None)
    b.ema = kw.get("ema", None)
    return b


def _call(fn, bank, hp=None, ws=FAKE * 16, ws_bytes=1 << 30, nb=1):
    lib = mb.raw_library()
    arr = (mb.CBank * 1)(bank)
    h = (hp or mb.Hparams()).to_c()
    return getattr(lib, fn)(arr, nb, ctypes.byref(h), ws, ws_bytes, None)


@pytest.mark.parametrize("fn", ["muon_step", "anvil_step"])
def test_validation_paths(fn):
    anvil = fn == "anvil_step"
    slow = FAKE + 0x3000 if anvil else None
    ok = dict(momentum_slow=slow)
    lib = mb.raw_library()
    h = mb.Hparams().to_c()
    assert getattr(lib, fn)(None, 1, ctypes.byref(h), FAKE, 1 << 30, None) == 1
    assert _call(fn, _bank(**ok), nb=0) == 2
    assert _call(fn, _bank(count=0, **ok)) == 2
    assert _call(fn, _bank(rows=-3, **ok)) == 2
    assert _call(fn, _bank(param=None, **ok)) == 1
    assert _call(fn, _bank(grad=None, **ok)) == 1
    assert _call(fn, _bank(param_dtype=5, **ok)) == 3
    assert _call(fn, _bank(grad=FAKE + 0x1004, **ok)) == 4
    assert _call(fn, _bank(**ok), hp=mb.Hparams(coeffs=[])) == 5
    assert _call(fn, _bank(**ok), hp=mb.Hparams(coeffs=[(1, 0, 0)] * 17)) == 5
    assert _call(fn, _bank(**ok), hp=mb.Hparams(coeffs=[(float("nan"), 0, 0)])) == 5
    assert _call(fn, _bank(**ok), hp=mb.Hparams(eps=-1.0)) == 5
    assert _call(fn, _bank(**ok), ws=None) == 6
    assert _call(fn, _bank(**ok), ws_bytes=1024) == 6
    assert _call(fn, _bank(param=FAKE, momentum=FAKE + 16, **ok)) == 9
    if anvil:
        assert _call(fn, _bank()) == 1  # momentum_slow missing
        assert _call(fn, _bank(**ok), hp=mb.Hparams(beta_slow=1.0)) == 5
    else:
        assert _call(fn, _bank(), hp=mb.Hparams(mu=1.5)) == 5
        assert _call(fn, _bank(ema=FAKE + 0x4000), hp=mb.Hparams(ema_beta=1.0)) == 5


@pytest.mark.parametrize("fn", ["muon_step", "anvil_step"])
def test_huge_shapes_rejected_without_overflow(fn):
    ok = dict(momentum_slow=FAKE + 0x3000 if fn == "anvil_step" else None)
    for kw in (dict(count=1 << 62), dict(rows=1 << 40), dict(cols=1 << 40),
               dict(count=1 << 30, rows=1 << 23, cols=1 << 23)):
        assert _call(fn, _bank(**kw, **ok)) == 2, kw


@pytest.mark.parametrize("fn", ["muon_step", "anvil_step"])
def test_buffers_of_different_banks_must_not_overlap(fn):
    """A buffer a step writes may not overlap one of another bank either."""
    lib = mb.raw_library()
    h = mb.Hparams().to_c()
    anvil = fn == "anvil_step"

    def bank(base):
        return _bank(param=base, grad=base + 0x1000, momentum=base + 0x2000,
                     momentum_slow=base + 0x3000 if anvil else None)

    def call(b0, b1):
        arr = (mb.CBank * 2)(b0, b1)
        return getattr(lib, fn)(arr, 2, ctypes.byref(h), FAKE * 16, 1 << 30, None)

    import torch
    if not torch.cuda.is_available():
        # valid arguments get past validation (and then fail on the missing
        # GPU); never run where kernels would launch on these fake addresses
        assert call(bank(FAKE), bank(FAKE + 0x8000)) == 7
    b1 = bank(FAKE + 0x8000)
    b1.momentum = FAKE  # bank 1's momentum on bank 0's parameters
    assert call(bank(FAKE), b1) == 9
    b1 = bank(FAKE + 0x8000)
    b1.param = FAKE + 0x2000 + 64  # inside bank 0's momentum
    assert call(bank(FAKE), b1) == 9


def test_valid_call_without_gpu_reports_cuda_error():
    """All arguments valid: the first CUDA call fails cleanly on a CPU host."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _call("muon_step", _bank()) == 7


def test_other_entry_points_validate():
    lib = mb.raw_library()
    h = mb.Hparams().to_c()
    assert lib.muon_orthogonalize(None, 1, FAKE, 1, 1, 8, 8, ctypes.byref(h), FAKE, 1 << 30, None) == 1
    assert lib.muon_orthogonalize(FAKE, 1, FAKE * 2, 1, 1, 0, 8, ctypes.byref(h), FAKE, 1 << 30, None) == 2
    assert lib.muon_orthogonalize(FAKE, 7, FAKE * 2, 1, 1, 8, 8, ctypes.byref(h), FAKE, 1 << 30, None) == 3
    assert lib.muon_orthogonalize(FAKE, 1, FAKE + 2, 1, 1, 8, 8, ctypes.byref(h), FAKE, 1 << 30, None) == 4
    assert lib.muon_orthogonalize(FAKE, 1, FAKE * 2, 1, 1, 8, 8, ctypes.byref(h), FAKE, 16, None) == 6
    assert lib.readout_blend(None, 1, FAKE, FAKE, 1, 10, 0.35, None) == 1
    assert lib.readout_blend(FAKE, 1, FAKE, FAKE, 1, 0, 0.35, None) == 2
    assert lib.readout_blend(FAKE, 1, FAKE + 4, FAKE, 1, 10, 0.35, None) == 4
    arr = (mb.CBank * 1)(_bank(ema=FAKE + 0x5000))
    assert lib.ema_update(arr, 1, 1.0, None) == 5
    assert lib.ema_update(None, 1, 0.5, None) == 1
    assert lib.muon_device_status(None, 4096, None, 0) == 1
    assert lib.muon_set_debug(3, 1.0) == 5
    assert lib.muon_set_debug(0, 0.0) == 0


@pytest.mark.slow
def test_debug_build_with_bounds_checks_compiles_and_exports():
    """`build.py --check` (-DMUON_CHECK) builds a library with every entry point
    and the extra status code (compiled here; no GPU needed)."""
    import importlib.util
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location(
        "_muon_b200_build", os.path.join(root, "muon_newton_schulz_05_b200", "build.py"))
    bld = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bld)
    path = bld.build(check=True)
    assert path.endswith("libmuonb200_check.so") and os.path.exists(path)
    lib = ctypes.CDLL(path)
    for name in mb.EXPORTED:
        getattr(lib, name)
    lib.muon_status_string.restype = ctypes.c_char_p
    assert b"MUON_ERR_BOUNDS" in lib.muon_status_string(10)
    assert mb.STATUS_NAMES[10] == "MUON_ERR_BOUNDS"


def test_checkpoint_average_betas_match_the_oracle():
    import oracle
    w = [0.5, 1.0, 3.0, 2.0, 1.5, 4.0]
    assert mb.checkpoint_average_betas(w) == pytest.approx(oracle.weighted_average_betas(w),
                                                           rel=0, abs=1e-15)
    assert mb.checkpoint_average_betas([2.0, 0.0, 1.0])[1] == 1.0  # zero weight: skip the call
    with pytest.raises(ValueError):
        mb.checkpoint_average_betas([0.0, 1.0])
    with pytest.raises(ValueError):
        mb.checkpoint_average_betas([1.0, -1.0])


HUGE = dict(count=500000, rows=4096, cols=4096)   # passes the per-bank shape check


def _plan_count(shapes, ns_steps):
    lib = mb.raw_library()
    f = lib.muon_chain_plan
    f.restype = ctypes.c_int64
    sh = (ctypes.c_int64 * (3 * len(shapes)))(*[v for s in shapes for v in s])
    return f(sh, len(shapes), ns_steps, None, ctypes.c_int64(0))


def test_totals_over_banks_and_steps_stay_in_32_bits():
    """Each bank can pass its own shape check while the chain's tile count over
    all phases and steps, or the elementwise passes' block count over all
    banks, would not fit the kernels' 32-bit indices: those are refused too."""
    one = (HUGE["count"], HUGE["rows"], HUGE["cols"])
    # 500000 x (136 Gram + 136 Poly + 256 Apply) tiles per step
    assert _plan_count([one], 5) == 5 * 500000 * 528
    assert _plan_count([one], 16) == -2
    # 500000 x 2048 momentum blocks per bank: two banks fit, three do not
    assert _plan_count([one] * 2, 1) == 2 * 500000 * 528
    assert _plan_count([one] * 3, 1) == -2


@pytest.mark.parametrize("fn", ["muon_step", "anvil_step"])
def test_step_refuses_totals_beyond_32_bits_before_the_workspace_check(fn):
    spaced = dict(param=1 << 48, grad=2 << 48, momentum=3 << 48,
                  momentum_slow=(4 << 48) if fn == "anvil_step" else None)
    bank = _bank(**HUGE, **spaced)
    q = (3.4445, -4.7750, 2.0315)
    assert _call(fn, bank, hp=mb.Hparams(coeffs=[q] * 5)) == 6        # only the workspace is short
    assert _call(fn, bank, hp=mb.Hparams(coeffs=[q] * 16)) == 2       # 16 steps: too many tiles


def test_orthogonalize_refuses_totals_beyond_32_bits():
    lib = mb.raw_library()
    q = (3.4445, -4.7750, 2.0315)
    for steps, want in ((5, 6), (16, 2)):
        h = mb.Hparams(coeffs=[q] * steps).to_c()
        st = lib.muon_orthogonalize(ctypes.c_void_p(1 << 48), mb.BF16, ctypes.c_void_p(2 << 48), mb.F32,
                                    ctypes.c_int64(HUGE["count"]), ctypes.c_int64(HUGE["rows"]),
                                    ctypes.c_int64(HUGE["cols"]), ctypes.byref(h),
                                    ctypes.c_void_p(FAKE), ctypes.c_size_t(1 << 30), None)
        assert st == want, (steps, st)


def test_ema_update_bounds_the_shape_before_multiplying():
    lib = mb.raw_library()
    for kw in (dict(count=1 << 40), dict(rows=1 << 40, cols=1 << 40), dict(count=0)):
        b = _bank(ema=FAKE + 0x4000, **kw)
        arr = (mb.CBank * 1)(b)
        assert lib.ema_update(arr, 1, ctypes.c_float(0.9), None) == 2, kw

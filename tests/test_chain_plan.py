"""The Newton-Schulz chain's tile list as the kernel decodes it, checked on the CPU.

`muon_chain_plan` runs the kernel's own tile decoder on the host. These tests
rebuild the list from its documented layout (step by step, phase by phase
Gram / Reduce / Poly / Apply, bank by bank, matrix by matrix; Apply tiles row
by row over the padded output, Gram and Poly tiles row by row over the upper
256-blocks, a split Gram's tile t of split s at t * ksplit + s with its own K
range) and check that the decoder puts every tile where the layout says and
that the operands each tile reads are the ones its product needs.
"""
import ctypes

import numpy as np
import pytest

import muon_newton_schulz_05_b200 as mb

GRAM, POLY, APPLY, REDUCE = 0, 1, 2, 3
ORDER = (GRAM, REDUCE, POLY, APPLY)


def _lib():
    lib = ctypes.CDLL(mb.LIB_PATH)
    f = lib.muon_chain_plan
    f.restype = ctypes.c_int64
    f.argtypes = [ctypes.POINTER(ctypes.c_int64), ctypes.c_int32, ctypes.c_int32,
                  ctypes.POINTER(ctypes.c_int32), ctypes.c_int64]
    return f


def chain_plan(shapes, ns_steps):
    f = _lib()
    sh = (ctypes.c_int64 * (3 * len(shapes)))(*[v for s in shapes for v in s])
    nt = f(sh, len(shapes), ns_steps, None, 0)
    assert nt > 0, nt
    til = np.zeros(13 * nt, dtype=np.int32)
    assert f(sh, len(shapes), ns_steps, til.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), til.size) == nt
    return til.reshape(-1, 13)


def pad(n):
    return (n + 255) // 256 * 256


def bank_geometry(count, rows, cols):
    Rp, Cp = pad(rows), pad(cols)
    tall = rows > cols
    rp = Cp if tall else Rp
    nb = rp // 256
    tiles_sym = nb * (nb + 1) // 2
    kg = (Rp if tall else Cp) // 64
    ksplit = 1
    if count * tiles_sym < 48 and kg * 64 >= 8 * rp:
        ksplit = max(1, min(16, kg // 32))
    kc = -(-kg // ksplit)
    if ksplit > 1:
        ksplit = -(-kg // kc)
    return dict(count=count, Rp=Rp, Cp=Cp, rp=rp, nb=nb, tall=tall, tiles_sym=tiles_sym,
                ksplit=ksplit, kc=kc, kg=kg, Mb=Rp // 256, Nb=Cp // 256,
                tiles_red=tiles_sym * 4 if ksplit > 1 else 0)


def sym_blocks(nb):
    return [(i, j) for i in range(nb) for j in range(i, nb)]


def expected_tiles(shapes, ns_steps):
    """(step, phase, bank, matrix, m0, n0, kb0, nkb) of every tile, in list order."""
    geos = [bank_geometry(*s) for s in shapes]
    out = []
    for k in range(ns_steps):
        for ph in ORDER:
            for b, g in enumerate(geos):
                for m in range(g["count"]):
                    if ph == APPLY:
                        kb = (g["Cp"] if g["tall"] else g["Rp"]) // 64
                        for i in range(g["Mb"]):
                            for j in range(g["Nb"]):
                                out.append((k, ph, b, m, 256 * i, 256 * j, 0, kb))
                    elif ph == POLY:
                        for i, j in sym_blocks(g["nb"]):
                            out.append((k, ph, b, m, 256 * i, 256 * j, 0, g["rp"] // 64))
                    elif ph == GRAM:
                        for i, j in sym_blocks(g["nb"]):
                            for s in range(g["ksplit"]):
                                kb0 = s * g["kc"] if g["ksplit"] > 1 else 0
                                nkb = min(g["kc"], g["kg"] - kb0) if g["ksplit"] > 1 else g["kg"]
                                out.append((k, ph, b, m, 256 * i, 256 * j, kb0, nkb))
                    else:
                        for _ in range(g["tiles_red"]):
                            out.append((k, ph, b, m, None, None, 0, 0))
    return out


SHAPES = {
    "gpt124m": [(48, 768, 768), (12, 768, 3072), (12, 3072, 768)],
    "square1024": [(64, 1024, 1024)],
    "anvil_readout": [(48, 768, 768), (12, 768, 3072), (12, 3072, 768), (1, 768, 50304)],
    "wide_2_5b": [(4, 2560, 2560), (2, 2560, 10240), (2, 10240, 2560)],
    "ragged": [(2, 7, 13), (1, 129, 257), (1, 257, 129), (3, 768, 1280), (1, 256, 256)],
    "odd_grid": [(3, 768, 1280), (5, 1280, 768)],
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_tiles_decode_to_the_documented_layout(name):
    shapes = SHAPES[name]
    til = chain_plan(shapes, 2)
    exp = expected_tiles(shapes, 2)
    assert len(exp) == len(til)
    for t, (e, got) in enumerate(zip(exp, til)):
        k, ph, b, m, m0, n0, kb0, nkb = e
        assert tuple(got[:4]) == (k, ph, b, m), (t, e, got)
        if ph != REDUCE:
            assert (got[4], got[5], got[6], got[7]) == (m0, n0, kb0, nkb), (t, e, got)


# map slots of the operands (the kernel's tensor-map table)
HI_K, HI_MN, A_K, B_K = (0, 1), (2, 3), 4, 5


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_each_tile_reads_the_operands_of_its_product(name):
    """Gram reads the current iterate twice (K-major for wide matrices,
    MN-major for tall ones), Poly reads A twice, Apply reads B and the
    iterate; all at the base row of the tile's own matrix, and the iterate
    buffer alternates with the step."""
    shapes = SHAPES[name]
    til = chain_plan(shapes, 3)
    geos = [bank_geometry(*s) for s in shapes]
    for t in til:
        k, ph, b, m = t[:4]
        if ph == REDUCE:
            continue
        g = geos[b]
        xbase, sbase = m * g["Rp"], m * g["rp"]
        cur = k & 1
        a_map, a_base, b_map, b_base = t[8], t[9], t[10], t[11]
        if ph == GRAM:
            want = HI_MN[cur] if g["tall"] else HI_K[cur]
            assert (a_map, b_map, a_base, b_base) == (want, want, xbase, xbase)
        elif ph == POLY:
            assert (a_map, b_map, a_base, b_base) == (A_K, A_K, sbase, sbase)
        elif g["tall"]:   # Y <- aY + Y B
            assert (a_map, a_base, b_map, b_base) == (HI_K[cur], xbase, B_K, sbase)
        else:             # X <- aX + B X
            assert (a_map, a_base, b_map, b_base) == (B_K, sbase, HI_MN[cur], xbase)


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_only_diagonal_symmetric_blocks_reuse_the_left_operand(name):
    """The right operand is skipped exactly on the diagonal blocks of Gram and
    Poly, where both sides are the same rows of the same matrix read the same
    way (same map, same base row, same first row)."""
    til = chain_plan(SHAPES[name], 2)
    for t in til:
        ph, m0, n0, same = t[1], t[4], t[5], t[12]
        want = int(ph in (GRAM, POLY) and m0 == n0)
        assert same == want, t
        if same:
            assert (t[8], t[9]) == (t[10], t[11])


def test_invalid_plans_are_refused():
    f = _lib()
    sh = (ctypes.c_int64 * 3)(1, 0, 5)
    assert f(sh, 1, 5, None, 0) < 0
    sh = (ctypes.c_int64 * 3)(1, 8, 8)
    assert f(sh, 1, 0, None, 0) < 0
    assert f(sh, 0, 5, None, 0) < 0

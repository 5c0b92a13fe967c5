"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Inputs come from muon_inputs (seeded, host-generated); the same bytes feed
both sides. Sizes span several 128x256 tiles plus ragged tails; the full
workloads are checked on sampled matrices (the oracle runs one matrix at a
time) and on every element for the elementwise buffers.
"""
import math

import numpy as np
import pytest
import torch

import muon_inputs as mi
import oracle
from _parity import (TOL_BUFFER, TOL_SV, TOL_UPDATE, buffer_ok, delta_ok, rel_fro,
                     bf16_ulp, sv_maxdiff, update_tols)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import muon_newton_schulz_05_b200 as mb
DEV = "cuda"
QUINTIC = mi.QUINTIC
CUBIC = mi.CUBIC


def f64(t):
    return oracle.as_f64(t.detach().cpu())


def orth_gpu(x, coeffs, out_dtype=torch.float32, eps=1e-7):
    cnt, R, C = x.shape
    ws = mb.alloc_workspace([(cnt, R, C)])
    out = torch.empty(cnt, R, C, dtype=out_dtype, device=DEV)
    mb.orthogonalize(x, out, mb.Hparams(coeffs=coeffs, eps=eps), ws)
    assert mb.device_status(ws) == 0
    return out


# ----------------------------------------------------------- orthogonalisation
SHAPES = [(1, 256, 256), (1, 256, 512), (1, 512, 256), (2, 7, 13), (2, 13, 7), (1, 1, 1),
          # a single row or column: X X^T is the squared norm, the result x / ||x|| * p(1)
          (1, 1, 777), (1, 777, 1),
          (1, 129, 257), (1, 257, 129), (2, 384, 640), (1, 768, 3072), (1, 3072, 768),
          # Gram K much longer than the Gram is wide: the product is split along K
          (1, 256, 8192), (1, 8192, 256), (1, 300, 20000)]
COEFFS = {
    "identity": ([(1.0, 0.0, 0.0)], 1e-5),
    "gram_only": ([(0.0, 1.0, 0.0)], 5e-3),
    "square_only": ([(0.0, 0.0, 1.0)], 5e-3),
    "cubic5": ([CUBIC] * 5, 5e-3),
    "quintic5": ([QUINTIC] * 5, TOL_UPDATE),
    "quintic6": ([QUINTIC] * 6, TOL_UPDATE),
    "schedule": ([(3.0, -3.2, 1.2), (2.0, -1.5, 0.5), (1.5, -0.5, 0.0)], 1e-2),
}


@pytest.mark.parametrize("shape", SHAPES, ids=[f"{c}x{r}x{k}" for c, r, k in SHAPES])
@pytest.mark.parametrize("cname", sorted(COEFFS))
def test_orthogonalize_matches_oracle(shape, cname):
    coeffs, tol = COEFFS[cname]
    cnt, R, C = shape
    g = mi.gaussian(cnt * R, C, seed=R * 1000 + C, sigma=1.0).reshape(cnt, R, C).to(torch.bfloat16)
    out = orth_gpu(g.to(DEV), coeffs).cpu()
    sv_tol = TOL_SV
    if min(R, C) < 32 and "quintic" in cname:
        tol, sv_tol = update_tols(R, C)
    for i in range(cnt):
        ref = oracle.orthogonalize(f64(g[i]), coeffs, 1e-7)
        got = f64(out[i])
        assert rel_fro(got, ref) <= tol, (i, rel_fro(got, ref))
        assert sv_maxdiff(got, ref) <= sv_tol


@pytest.mark.parametrize("rank", [1, 64])
@pytest.mark.parametrize("shape", [(768, 768), (768, 3072), (3072, 768)])
def test_orthogonalize_low_rank_gradients(rank, shape):
    """Gradients of low rank (x^T dy over `rank` rows, as one small batch
    gives): in their null space only the a X term acts, so the iterate's
    rounding noise grows by a per step unless X is carried to more than bf16
    precision through every step."""
    R, C = shape
    g = torch.Generator().manual_seed(rank * 7 + R)
    x = torch.randn(rank, R, generator=g, dtype=torch.float64)
    dy = torch.randn(rank, C, generator=g, dtype=torch.float64)
    u = (x.T @ dy).to(torch.bfloat16)[None]
    for coeffs in ([QUINTIC] * 5, [QUINTIC] * 6):
        out = orth_gpu(u.to(DEV), coeffs).cpu()
        ref = oracle.orthogonalize(f64(u[0]), coeffs, 1e-7)
        assert rel_fro(f64(out[0]), ref) <= TOL_UPDATE, (len(coeffs), rel_fro(f64(out[0]), ref))
        assert sv_maxdiff(f64(out[0]), ref) <= TOL_SV


@pytest.mark.parametrize("shape", [(1, 129, 257), (1, 768, 768), (1, 257, 129), (1, 256, 8192), (2, 384, 640)])
def test_sixteen_steps_each_with_its_own_coefficients(shape):
    """The most steps a call takes (16), each with different coefficients
    (five quintic, then eleven convergent cubic variants with a + b = 1), so a
    coefficient read from the wrong step shows: the same schedule shifted by
    one step is 0.3 away from the oracle."""
    s16 = [QUINTIC] * 5 + [(1.5 + 0.01 * j, -0.5 - 0.01 * j, 0.0) for j in range(11)]
    cnt, R, C = shape
    g = mi.gaussian(cnt * R, C, seed=R * 1000 + C, sigma=1.0).reshape(cnt, R, C).to(torch.bfloat16)
    out = orth_gpu(g.to(DEV), s16).cpu()
    for i in range(cnt):
        ref = oracle.orthogonalize(f64(g[i]), s16, 1e-7)
        assert rel_fro(f64(out[i]), ref) <= TOL_UPDATE, (i, rel_fro(f64(out[i]), ref))
        assert sv_maxdiff(f64(out[i]), ref) <= TOL_SV


def test_many_matrices_in_one_call():
    """Hundreds of matrices in one call (thousands of tiles and per-matrix
    counters in one persistent launch), wide and tall, every one checked.
    The inputs are spiked like the benchmark banks' gradients (N(0, 1e-3^2)
    plus a rank-4 spike at 10x RMS; a replay of the kernel's rounding puts
    them at about half the tolerance; plain Gaussian matrices of this size
    sit at 0.85-0.95 of it)."""
    for base, cnt, R, C in ((1000, 300, 64, 128), (2000, 150, 128, 64)):
        x = torch.stack([mi.spiked_gaussian(R, C, base + i, 1e-3, 4, 10.0) for i in range(cnt)])
        out = orth_gpu(x.to(DEV), [QUINTIC] * 5).cpu()
        for i in range(cnt):
            ref = oracle.orthogonalize(f64(x[i]), [QUINTIC] * 5, 1e-7)
            assert rel_fro(f64(out[i]), ref) <= TOL_UPDATE, (R, C, i, rel_fro(f64(out[i]), ref))
            assert sv_maxdiff(f64(out[i]), ref) <= TOL_SV


def test_orthogonalize_bf16_output_and_fp32_input():
    x = mi.spiked_gaussian(768, 768, 5, 1e-3, 4, 10.0)[None].to(DEV)
    out = orth_gpu(x, [QUINTIC] * 5, out_dtype=torch.bfloat16)
    ref = oracle.orthogonalize(f64(x[0]), [QUINTIC] * 5, 1e-7)
    assert rel_fro(f64(out[0]), ref) <= TOL_UPDATE
    assert sv_maxdiff(f64(out[0]), ref) <= TOL_SV


def test_zero_gradient_gives_zero_update():
    x = torch.zeros(2, 256, 384, dtype=torch.bfloat16, device=DEV)
    out = orth_gpu(x, [QUINTIC] * 5)
    assert torch.count_nonzero(out) == 0


# ---------------------------------------------------------------- Muon steps
def _muon_run(w, steps, check_steps, sample, hp_override=None):
    """Run `steps` Muon steps of workload w on the GPU; at check_steps compare
    the momentum (all elements), the update (sampled matrices, through the
    NS of the GPU's own U) and the parameter step (sampled, teacher-forced)."""
    hp = dict(w.hp)
    if hp_override:
        hp.update(hp_override)
    banks = []
    for b, spec in enumerate(w.banks):
        th = mi.make_params(w, b).to(DEV)
        M = torch.zeros(th.shape, dtype=torch.float32, device=DEV)
        banks.append(mb.Bank(th, None, M))
    ws = mb.alloc_workspace([bk.shape for bk in banks])
    H = mb.Hparams.from_dict(hp)
    for step in range(steps):
        grads = [mi.make_grads(w, b, step) for b in range(len(w.banks))]
        check = step in check_steps
        if check:
            old = [(bk.param.clone(), bk.momentum.clone()) for bk in banks]
        for bk, g in zip(banks, grads):
            bk.grad = g.to(DEV)
        mb.muon_step(banks, H, ws)
        torch.cuda.synchronize()
        assert mb.device_status(ws) == 0
        if not check:
            continue
        for b, bk in enumerate(banks):
            th0, M0 = old[b]
            G = grads[b]
            # momentum on every element
            sgd = bool(hp.get("sgd_momentum"))
            upd = oracle.momentum_update_sgd if sgd else oracle.momentum_update
            look = oracle.nesterov_lookahead_sgd if sgd else oracle.nesterov_lookahead
            Mref = upd(f64(M0), f64(G), hp["mu"])
            ok, r = buffer_ok(f64(bk.momentum), Mref, TOL_BUFFER)
            assert ok, ("momentum", b, step, r)
            R, C = bk.shape[1:]
            s = oracle.shape_scale(R, C)
            tol_o, tol_sv = update_tols(R, C)
            for i in sample(b, bk.shape[0]):
                U = look(Mref[i], f64(G[i]), hp["mu"], bool(hp["nesterov"]))
                O = oracle.orthogonalize(U, hp["coeffs"], hp["eps"])
                # the NS path on the GPU's own U
                Ug = torch.from_numpy(U.astype(np.float32))[None].to(DEV)
                Og = f64(orth_gpu(Ug, hp["coeffs"])[0])
                assert rel_fro(Og, O) <= tol_o, ("O", b, i, step, rel_fro(Og, O))
                assert sv_maxdiff(Og, O) <= tol_sv
                # parameter step (teacher-forced on the GPU's theta_old)
                t0 = f64(th0[i])
                dref = oracle.decoupled_update(t0, O, hp["lr"], hp["weight_decay"], s) - t0
                ok, r = delta_ok(t0, f64(bk.param[i]), dref, w.param_dtype, tol_o)
                assert ok, ("delta", b, i, step, r)
    return banks


def test_single_matrix_fp32_three_steps():
    w = mi.workloads()[1]
    _muon_run(w, 3, {0, 1, 2}, lambda b, n: range(n))


def test_gpt124m_bank_ten_steps():
    w = mi.workloads()[2]
    _muon_run(w, w.steps, {0, 4, 9}, lambda b, n: [0, n - 1])


def test_square_1024_bank_with_decay():
    w = mi.workloads()[3]
    _muon_run(w, w.steps, {0, 12, w.steps - 1}, lambda b, n: [0, 37, n - 1])


def test_sgd_form_momentum_flag():
    w = mi.custom_workload([(4, 512, 768), (2, 768, 512)],
                           dict(lr=0.02, mu=0.9, weight_decay=0.05, nesterov=1,
                                coeffs=[QUINTIC] * 5, eps=1e-7, sgd_momentum=1), cid=93)
    _muon_run(w, 3, {0, 2}, lambda b, n: [0, n - 1])


def test_ragged_bank_mix():
    w = mi.custom_workload([(3, 200, 72), (2, 72, 200), (1, 1000, 1000), (2, 8, 1)],
                           dict(lr=0.03, mu=0.9, weight_decay=0.1, nesterov=1,
                                coeffs=[QUINTIC] * 5, eps=1e-7),
                           param_dtype="f32", grad_dtype="bf16")
    _muon_run(w, 2, {0, 1}, lambda b, n: range(n))


# ---------------------------------------------------------------- ANVIL + EMA
def test_anvil_steps_ema_and_readout_blend():
    w = mi.workloads()[5]
    hp = w.hp
    banks = []
    for b in range(len(w.banks)):
        th = mi.make_params(w, b).to(DEV)
        z = torch.zeros(th.shape, dtype=torch.float32, device=DEV)
        banks.append(mb.Bank(th, None, z.clone(), z.clone(), th.float().clone()))
    ws = mb.alloc_workspace([bk.shape for bk in banks])
    H = mb.Hparams.from_dict(hp)
    steps = w.steps  # 50: the averaging window of the workload
    checked = {0, 1, steps // 2, steps - 1}
    for step in range(steps):
        grads = [mi.make_grads(w, b, step) for b in range(len(w.banks))]
        check = step in checked
        if check:
            old = [(bk.param.clone(), bk.momentum.clone(), bk.momentum_slow.clone(), bk.ema.clone())
                   for bk in banks]
        for bk, g in zip(banks, grads):
            bk.grad = g.to(DEV)
        mb.anvil_step(banks, H, ws)
        torch.cuda.synchronize()
        assert mb.device_status(ws) == 0
        if not check:
            continue
        for b, bk in enumerate(banks):
            th0, Mf0, Ms0, E0 = old[b]
            G = f64(grads[b])
            Mf = oracle.momentum_update(f64(Mf0), G, hp["beta_fast"])
            Ms = oracle.momentum_update(f64(Ms0), G, hp["beta_slow"])
            assert buffer_ok(f64(bk.momentum), Mf)[0]
            assert buffer_ok(f64(bk.momentum_slow), Ms)[0]
            # EMA teacher-forced on the GPU's stored parameters
            Eref = oracle.ema_update(f64(E0), f64(bk.param), hp["ema_beta"])
            ok, r = buffer_ok(f64(bk.ema), Eref)
            assert ok, ("ema", b, r)
            if step != steps - 1:
                continue
            R, C = bk.shape[1:]
            picks = [0] if bk.shape[0] == 1 else [0, bk.shape[0] - 1]
            for i in picks:
                O = oracle.orthogonalize(Mf[i], hp["coeffs"], hp["eps"])
                mask = oracle.cautious_mask(O, Ms[i])
                t0 = f64(th0[i])
                dref = oracle.cautious_update(t0, O, mask, hp["lr"], hp["weight_decay"],
                                              oracle.shape_scale(R, C)) - t0
                ok, r = delta_ok(t0, f64(bk.param[i]), dref, "bf16")
                assert ok, ("anvil delta", b, i, r)
                # six polynomial applications on the GPU's own fast momentum
                Og = f64(orth_gpu(bk.momentum[i:i + 1].clone(), hp["coeffs"])[0])
                assert rel_fro(Og, O) <= TOL_UPDATE, ("anvil O", b, i, rel_fro(Og, O))
                assert sv_maxdiff(Og, O) <= TOL_SV
    # readout blend on the 768 x 50304 readout
    rd = banks[-1]
    out = torch.empty_like(rd.param)
    mb.readout_blend(rd.param, rd.ema, out, hp["readout_final_weight"])
    ref = oracle.readout_blend(f64(rd.param), f64(rd.ema), hp["readout_final_weight"])
    assert np.array_equal(f64(out), oracle.round_to_bf16(ref)) or rel_fro(f64(out), ref) < 4e-3


def test_anvil_mask_decisions_agree_where_unambiguous():
    """Mask decisions compared where |O * M_slow| is not tiny (both sides must
    agree there); elsewhere either decision is valid."""
    R, C = 512, 768
    th = (mi.gaussian(R, C, 1, 0.02)[None]).to(DEV)
    G = mi.spiked_gaussian(R, C, 2, 1e-3, 4, 10.0)[None].to(torch.bfloat16)
    Ms0 = mi.gaussian(R, C, 3, 1e-3)[None]
    hp = dict(lr=0.05, beta_fast=0.9, beta_slow=0.99, weight_decay=0.5, eps=1e-7,
              coeffs=[QUINTIC] * 6)
    bank = mb.Bank(th.clone(), G.to(DEV), torch.zeros(1, R, C, device=DEV), Ms0.clone().to(DEV))
    ws = mb.alloc_workspace([bank.shape])
    mb.anvil_step([bank], mb.Hparams.from_dict(hp), ws)
    torch.cuda.synchronize()
    Mf = oracle.momentum_update(np.zeros((R, C)), f64(G[0]), 0.9)
    Ms = oracle.momentum_update(f64(Ms0[0]), f64(G[0]), 0.99)
    O = oracle.orthogonalize(Mf, hp["coeffs"], 1e-7)
    mask = oracle.cautious_mask(O, Ms)
    t0 = f64(th[0])
    lr, wd, s = 0.05, 0.5, 1.0
    # recover the GPU's decay decision: theta_new = t0 - lr wd m t0 - lr s O.
    # O must be the step's own: the orthogonalisation of the GPU's fast momentum
    # reproduces it bit for bit, while an input one fp32 ulp away re-draws the
    # ~1 % bf16 rounding error (elementwise up to ~8 % of rms(O) in the tails).
    Og = f64(orth_gpu(bank.momentum.clone(), hp["coeffs"])[0])
    pred_nodecay = t0 - lr * s * Og
    pred_decay = t0 - lr * wd * t0 - lr * s * Og
    got = f64(bank.param[0])
    decided = np.where(np.abs(got - pred_decay) < np.abs(got - pred_nodecay), 1.0, 0.0)
    # O carries ~1 % relative error; its sign is certain where |O| is well
    # above that, and M_slow is fp32-exact against the oracle
    rms = lambda a: np.sqrt(np.mean(a * a))
    sure = (np.abs(O) > 0.2 * rms(O)) & (np.abs(Ms) > 1e-3 * rms(Ms))
    # the decision is recoverable only where the decay term is well above the
    # bf16 rounding of the stored parameter
    sure &= lr * wd * np.abs(t0) > 3.0 * bf16_ulp(got)
    assert sure.sum() > 0.3 * sure.size, sure.sum()
    bad = int(np.sum(decided[sure] != mask[sure]))
    assert bad == 0, (bad, int(sure.sum()))


def test_standalone_ema_update():
    th = mi.gaussian(3 * 37, 91, 9, 0.02).reshape(3, 37, 91).to(torch.bfloat16).to(DEV)
    e = mi.gaussian(3 * 37, 91, 10, 0.02).reshape(3, 37, 91).to(DEV)
    e0 = e.clone()
    mb.ema_update([mb.Bank(th, th, torch.zeros(3, 37, 91, device=DEV), None, e)], 0.9)
    torch.cuda.synchronize()
    ok, r = buffer_ok(f64(e), oracle.ema_update(f64(e0), f64(th), 0.9))
    assert ok, r


# --------------------------------------------------- determinism, resume, graph
def _small_bank(seed=0):
    w = mi.custom_workload([(4, 256, 640), (2, 640, 256)],
                           dict(lr=0.02, mu=0.95, weight_decay=0.01, nesterov=1,
                                coeffs=[QUINTIC] * 5, eps=1e-7), cid=91)
    banks = []
    for b in range(2):
        th = mi.make_params(w, b).to(DEV)
        banks.append(mb.Bank(th, None, torch.zeros(th.shape, device=DEV), None,
                             th.float().clone()))
    return w, banks


def _run(w, banks, ws, steps, start=0):
    H = mb.Hparams.from_dict(dict(w.hp, ema_beta=0.99))
    for s in range(start, start + steps):
        for b, bk in enumerate(banks):
            bk.grad = mi.make_grads(w, b, s).to(DEV)
        mb.muon_step(banks, H, ws)
    torch.cuda.synchronize()


def test_deterministic_and_resume_bitwise():
    w, b1 = _small_bank()
    ws = mb.alloc_workspace([b.shape for b in b1])
    _run(w, b1, ws, 4)
    _, b2 = _small_bank()
    ws2 = mb.alloc_workspace([b.shape for b in b2])
    _run(w, b2, ws2, 2)
    # "checkpoint": copy the state to fresh tensors and a fresh workspace
    b3 = [mb.Bank(b.param.clone(), None, b.momentum.clone(), None, b.ema.clone()) for b in b2]
    ws3 = mb.alloc_workspace([b.shape for b in b3])
    _run(w, b3, ws3, 2, start=2)
    for x, y in zip(b1, b3):
        assert torch.equal(x.param, y.param)
        assert torch.equal(x.momentum, y.momentum)
        assert torch.equal(x.ema, y.ema)


def test_cuda_graph_capture_replays_the_step():
    w, b1 = _small_bank()
    _, b2 = _small_bank()
    ws1 = mb.alloc_workspace([b.shape for b in b1])
    ws2 = mb.alloc_workspace([b.shape for b in b2])
    H = mb.Hparams.from_dict(w.hp)
    for b, (x, y) in enumerate(zip(b1, b2)):
        g = mi.make_grads(w, b, 0).to(DEV)
        x.grad, y.grad = g, g.clone()
    mb.muon_step(b1, H, ws1)  # eager
    mb.muon_step(b2, H, ws2)  # warm-up of the second set so both take two steps
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        graph.capture_begin()
        mb.muon_step(b2, H, ws2, stream=s)
        graph.capture_end()
    graph.replay()
    mb.muon_step(b1, H, ws1)
    torch.cuda.synchronize()
    for x, y in zip(b1, b2):
        assert torch.equal(x.param, y.param)
        assert torch.equal(x.momentum, y.momentum)


def test_bounded_wait_timeout_is_reported_and_recovers():
    x = mi.gaussian(256, 512, 4, 1.0)[None].to(torch.bfloat16).to(DEV)
    ws = mb.alloc_workspace([(1, 256, 512)])
    out = torch.empty(1, 256, 512, device=DEV)
    H = mb.Hparams(coeffs=[QUINTIC] * 2)
    try:
        mb.set_debug(1, 0.25)
        mb.orthogonalize(x, out, H, ws)
        assert mb.device_status(ws, clear=True) == 8
    finally:
        mb.set_debug(0, 0.0)
    mb.orthogonalize(x, out, H, ws)
    assert mb.device_status(ws) == 0
    ref = oracle.orthogonalize(f64(x[0]), [QUINTIC] * 2, 1e-7)
    assert rel_fro(f64(out[0]), ref) < TOL_UPDATE


def test_timeout_in_a_step_leaves_params_and_ema_unchanged():
    """A bounded wait that runs out inside a step (the test hook withholds one
    operand stage) is reported, and the step writes no parameter and no EMA;
    the momenta advanced once (their pass runs before the chain). While the
    status word holds the error, further steps change nothing at all; once
    it is cleared, steps run again and match the oracle."""
    w, banks = _small_bank()
    ws = mb.alloc_workspace([b.shape for b in banks])
    H = mb.Hparams.from_dict(dict(w.hp, ema_beta=0.99))
    grads = [mi.make_grads(w, b, 0) for b in range(2)]
    for bk, g in zip(banks, grads):
        bk.grad = g.to(DEV)
    p0 = [b.param.clone() for b in banks]
    e0 = [b.ema.clone() for b in banks]
    try:
        mb.set_debug(1, 0.25)
        mb.muon_step(banks, H, ws)
        assert mb.device_status(ws) == 8
    finally:
        mb.set_debug(0, 0.0)
    for b, bk in enumerate(banks):
        assert torch.equal(bk.param, p0[b]) and torch.equal(bk.ema, e0[b])
        Mref = oracle.momentum_update(np.zeros(bk.momentum.shape), f64(grads[b]), w.hp["mu"])
        assert buffer_ok(f64(bk.momentum), Mref)[0]
    m1 = [b.momentum.clone() for b in banks]
    mb.muon_step(banks, H, ws)             # the error is still recorded: a no-op
    assert mb.device_status(ws, clear=True) == 8
    for b, bk in enumerate(banks):
        assert torch.equal(bk.param, p0[b]) and torch.equal(bk.ema, e0[b])
        assert torch.equal(bk.momentum, m1[b])
    mb.muon_step(banks, H, ws)             # cleared: a normal step
    torch.cuda.synchronize()
    assert mb.device_status(ws) == 0
    for b, bk in enumerate(banks):
        R, C = bk.shape[1:]
        G = f64(grads[b][0])
        Mref = oracle.momentum_update(f64(m1[b][0]), G, w.hp["mu"])
        U = oracle.nesterov_lookahead(Mref, G, w.hp["mu"], True)
        O = oracle.orthogonalize(U, w.hp["coeffs"], w.hp["eps"])
        t0 = f64(p0[b][0])
        dref = oracle.decoupled_update(t0, O, w.hp["lr"], w.hp["weight_decay"],
                                       oracle.shape_scale(R, C)) - t0
        ok, r = delta_ok(t0, f64(bk.param[0]), dref, "bf16")
        assert ok, r


def test_weighted_checkpoint_average_through_ema_update():
    """Weighted checkpoint average ("qlabs-eng/slowrun", leaderboard: weighted
    checkpoint averaging) as ema_update with the running beta of each
    checkpoint, against the oracle's sum w_i theta_i / sum w_i."""
    n, shape = 7, (3, 129, 200)
    weights = [0.5, 1.0, 3.0, 0.0, 2.0, 1.5, 4.0]
    thetas = [mi.gaussian(shape[0] * shape[1], shape[2], 500 + i, 0.02).reshape(shape)
              .to(torch.bfloat16) for i in range(n)]
    th = thetas[0].to(DEV)
    avg = torch.zeros(shape, device=DEV)
    bank = mb.Bank(th, th, torch.zeros(shape, device=DEV), None, avg)
    for wt, w_i, beta in zip(thetas, weights, mb.checkpoint_average_betas(weights)):
        if w_i == 0.0:
            continue  # no weight: the checkpoint does not enter the average
        th.copy_(wt.to(DEV))
        mb.ema_update([bank], beta)
    torch.cuda.synchronize()
    ref = oracle.weighted_average([f64(t) for t in thetas], weights)
    ok, r = buffer_ok(f64(avg), ref)
    assert ok, r


def test_invalid_arguments_launch_nothing():
    x = torch.zeros(1, 64, 64, dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(mb.MuonError) as e:
        mb.orthogonalize(x, torch.empty(1, 64, 64, device=DEV), mb.Hparams(), ws)
    assert e.value.code == 6


# ------------------------------------------------------- full-size workloads
@pytest.mark.slow
def test_transformer_2p5b_bank_sampled():
    """The 2.5B bank (192 matrices, 2,516,582,400 parameters) for one step,
    in the same launch configuration as the benchmark; momentum, update and
    step checked on one matrix of each shape (first and last layers)."""
    w = mi.workloads()[4]
    hp = w.hp
    banks, grads_host = [], []
    for b, spec in enumerate(w.banks):
        th = mi.make_params(w, b).to(DEV)
        g = mi.make_grads(w, b, 0)
        grads_host.append(g)
        banks.append(mb.Bank(th, g.to(DEV), torch.zeros(th.shape, device=DEV)))
    ws = mb.alloc_workspace([bk.shape for bk in banks])
    th0 = [bk.param.clone() for bk in banks]
    mb.muon_step(banks, mb.Hparams.from_dict(hp), ws)
    torch.cuda.synchronize()
    assert mb.device_status(ws) == 0
    picks = {0: [127], 1: [0], 2: [31]}
    for b, bk in enumerate(banks):
        R, C = bk.shape[1:]
        for i in picks[b]:
            G = f64(grads_host[b][i])
            Mref = oracle.momentum_update(np.zeros_like(G), G, hp["mu"])
            assert buffer_ok(f64(bk.momentum[i]), Mref)[0]
            U = oracle.nesterov_lookahead(Mref, G, hp["mu"], True)
            O = oracle.orthogonalize(U, hp["coeffs"], hp["eps"])
            t0 = f64(th0[b][i])
            dref = oracle.decoupled_update(t0, O, hp["lr"], hp["weight_decay"],
                                           oracle.shape_scale(R, C)) - t0
            ok, r = delta_ok(t0, f64(bk.param[i]), dref, "bf16")
            assert ok, ("delta", b, i, r)
            # the Newton-Schulz chain at this size on the same U (one matrix,
            # the benchmark's kernel): relative Frobenius and singular values
            Ug = torch.from_numpy(U.astype(np.float32))[None].to(DEV)
            Og = f64(orth_gpu(Ug, hp["coeffs"])[0])
            assert rel_fro(Og, O) <= TOL_UPDATE, ("O", b, i, rel_fro(Og, O))
            assert sv_maxdiff(Og, O) <= TOL_SV, ("singular values", b, i)

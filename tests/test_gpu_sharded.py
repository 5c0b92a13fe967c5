"""Owner-sharded data-parallel step on the GPU: one NCCL rank, the library's step.

With one rank the reduce-scatter averages over one gradient and every matrix
is owned locally. Each step is checked two ways: against a direct call of the
library on the whole bank (bitwise: the sharded plumbing must not change a
bit), and against the CPU oracle on the rank's mean gradient (here its own):
every momentum element, the parameter step of sampled matrices and, with
fp32 parameters, the orthogonalised update and its singular values. The
multi-rank exchange is covered on CPU with gloo.
"""
import socket

import pytest
import torch

from _oracle_checks import check_anvil_step, check_muon_step, hp_dict

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SHAPES = [(6, 768, 768), (2, 768, 3072), (2, 3072, 768)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group():
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, device_id=torch.device(DEV))
    yield dist
    dist.destroy_process_group()


def _bank(seed, scale=1.0):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return [torch.randn(c, r, k, generator=g, device=DEV) * scale for c, r, k in SHAPES]


def _hparams(variant):
    import muon_newton_schulz_05_b200 as mb
    if variant == "anvil":
        return mb.Hparams(lr=0.05, weight_decay=0.1, coeffs=[(3.4445, -4.7750, 2.0315)] * 6,
                          beta_fast=0.9, beta_slow=0.99, ema_beta=0.99)
    return mb.Hparams(lr=0.05, mu=0.95, weight_decay=0.01, nesterov=True)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("variant", ["muon", "anvil"])
def test_sharded_single_rank_equals_direct_step_and_oracle(nccl_group, variant, dtype):
    import muon_newton_schulz_05_b200 as mb
    from muon_newton_schulz_05_b200.sharded import ShardedMuon
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    hp = _hparams(variant)
    ohp = hp_dict(hp)
    params = [p.to(tdt) for p in _bank(1, 0.02)]
    ref = [p.clone() for p in params]
    opt = ShardedMuon(SHAPES, tdt, torch.bfloat16, variant=variant, device=DEV,
                      buckets=[[1, 2], [0]], ema=(variant == "anvil"))
    mom = [torch.zeros(c, r, k, device=DEV) for c, r, k in SHAPES]
    slow = [torch.zeros_like(m) for m in mom] if variant == "anvil" else [None] * 3
    ema = [p.float().clone() for p in ref] if variant == "anvil" else [None] * 3
    banks = [mb.Bank(ref[b], None, mom[b], slow[b], ema[b]) for b in range(3)]
    ws = mb.alloc_workspace([bk.shape for bk in banks])
    for s in range(3):
        grads = [g.to(torch.bfloat16) for g in _bank(100 + s)]
        before = [(p.clone(), m.clone(), None if sl is None else sl.clone())
                  for p, m, sl in zip(params, mom, slow)]
        opt.step(params, grads, hp)
        for b in range(3):
            banks[b].grad = grads[b]
        (mb.anvil_step if variant == "anvil" else mb.muon_step)(banks, hp, ws)
        torch.cuda.synchronize()
        for b in range(3):
            assert torch.equal(params[b], ref[b]), (s, b)
        if s == 1:  # the oracle on this step (the rank's mean gradient is its own)
            for b in range(3):
                picks = [0, SHAPES[b][0] - 1]
                th0, m0, sl0 = before[b]
                if variant == "anvil":
                    check_anvil_step(th0, params[b], grads[b], m0, mom[b], sl0, slow[b], ohp,
                                     picks, dtype)
                else:
                    check_muon_step(th0, params[b], grads[b], m0, mom[b], ohp, picks, dtype)
    assert mb.device_status(ws) == 0
    assert all(mb.device_status(w) == 0 for w in opt.workspaces if w is not None)
    for b in range(3):
        # one rank owns every matrix of a bank, in order
        k, j = next((k, j) for k, bk in enumerate(opt.plan.buckets) for j, x in enumerate(bk.banks)
                    if x == b)
        assert torch.equal(opt.momentum[k][j], mom[b])
        if variant == "anvil":
            assert torch.equal(opt.momentum_slow[k][j], slow[b])
            assert torch.equal(opt.ema[k][j], ema[b])
    if variant == "anvil":
        out = [torch.zeros(c, r, k, device=DEV) for c, r, k in SHAPES]
        opt.gather_ema(out)
        for b in range(3):
            assert torch.equal(out[b], ema[b])


@pytest.mark.parametrize("per_bank", [False, True])
@pytest.mark.parametrize("variant", ["muon", "anvil"])
def test_bank_storage_single_rank_equals_direct_step_and_oracle(nccl_group, variant, per_bank):
    """ShardedBankMuon (owner-ordered bank storage, in-place reduce-scatter and
    all-gather) on one rank: bitwise a direct call of the library, and the
    oracle on the second step (fp32 parameters: O recovered from the step)."""
    import muon_newton_schulz_05_b200 as mb
    from muon_newton_schulz_05_b200.sharded import ShardedBankMuon
    hp = _hparams(variant)
    ohp = hp_dict(hp)
    opt = ShardedBankMuon(SHAPES, torch.float32, torch.bfloat16, variant=variant, device=DEV,
                          ema=(variant == "anvil"), per_bank=per_bank)
    init = _bank(2, 0.02)
    for p, p0 in zip(opt.params, init):
        p.copy_(p0)
    ref = [p.clone() for p in init]
    mom = [torch.zeros(c, r, k, device=DEV) for c, r, k in SHAPES]
    slow = [torch.zeros_like(m) for m in mom] if variant == "anvil" else [None] * 3
    ema = [p.clone() for p in ref] if variant == "anvil" else [None] * 3
    banks = [mb.Bank(ref[b], None, mom[b], slow[b], ema[b]) for b in range(3)]
    ws = mb.alloc_workspace([bk.shape for bk in banks])
    for s in range(3):
        grads = [g.to(torch.bfloat16) for g in _bank(200 + s)]
        for g, g0 in zip(opt.grads, grads):
            g.copy_(g0)
        before = [(p.clone(), m.clone(), None if sl is None else sl.clone())
                  for p, m, sl in zip(opt.params, mom, slow)]
        opt.step(hp)
        for b in range(3):
            banks[b].grad = grads[b]
        (mb.anvil_step if variant == "anvil" else mb.muon_step)(banks, hp, ws)
        torch.cuda.synchronize()
        for b in range(3):
            assert torch.equal(opt.params[b], ref[b]), (s, b)
            assert torch.equal(opt.momentum[b], mom[b])
        if s == 1:
            for b in range(3):
                picks = [0, SHAPES[b][0] - 1]
                th0, m0, sl0 = before[b]
                if variant == "anvil":
                    check_anvil_step(th0, opt.params[b], grads[b], m0, mom[b], sl0, slow[b], ohp,
                                     picks, "f32")
                else:
                    check_muon_step(th0, opt.params[b], grads[b], m0, mom[b], ohp, picks, "f32")
    assert mb.device_status(ws) == 0 and opt.device_status() == 0
    if variant == "anvil":
        out = [torch.zeros(c, r, k, device=DEV) for c, r, k in SHAPES]
        opt.gather_ema(out)
        for b in range(3):
            assert torch.equal(out[b], ema[b])

"""Owner-sharded data-parallel step on the GPU: one NCCL rank, the library's step.

With one rank the reduce-scatter averages over one gradient and every matrix
is owned locally, so the sharded step (bucketed collectives, owner step,
all-gather, unpack) must give exactly what a direct call of the library on
the whole bank gives. The multi-rank exchange is covered on CPU with gloo.
"""
import socket

import pytest
import torch

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


def _bank(seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return [torch.randn(c, r, k, generator=g, device=DEV) for c, r, k in SHAPES]


@pytest.mark.parametrize("variant", ["muon", "anvil"])
def test_sharded_single_rank_equals_direct_step(nccl_group, variant):
    import muon_newton_schulz_05_b200 as mb
    from muon_newton_schulz_05_b200.sharded import ShardedMuon
    if variant == "anvil":
        hp = mb.Hparams(lr=0.05, weight_decay=0.1, coeffs=[(3.4445, -4.7750, 2.0315)] * 6,
                        beta_fast=0.9, beta_slow=0.99, ema_beta=0.99)
    else:
        hp = mb.Hparams(lr=0.05, mu=0.95, weight_decay=0.01, nesterov=True)
    params = [p.to(torch.bfloat16) for p in _bank(1)]
    ref = [p.clone() for p in params]
    opt = ShardedMuon(SHAPES, torch.bfloat16, torch.bfloat16, variant=variant, device=DEV,
                      buckets=[[1, 2], [0]], ema=(variant == "anvil"))
    mom = [torch.zeros(c, r, k, device=DEV) for c, r, k in SHAPES]
    slow = [torch.zeros_like(m) for m in mom] if variant == "anvil" else [None] * 3
    ema = [p.float() for p in ref] if variant == "anvil" else [None] * 3
    banks = [mb.Bank(ref[b], None, mom[b], slow[b], ema[b]) for b in range(3)]
    ws = mb.alloc_workspace([bk.shape for bk in banks])
    for s in range(3):
        grads = [g.to(torch.bfloat16) for g in _bank(100 + s)]
        opt.step(params, grads, hp)
        for b in range(3):
            banks[b].grad = grads[b]
        (mb.anvil_step if variant == "anvil" else mb.muon_step)(banks, hp, ws)
    torch.cuda.synchronize()
    assert mb.device_status(ws) == 0
    assert all(mb.device_status(w) == 0 for w in opt.workspaces)
    for b in range(3):
        assert torch.equal(params[b], ref[b]), b
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

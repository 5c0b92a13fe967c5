"""Owner-sharded data-parallel Muon on CPU: gloo ranks, the oracle as the local step.

The collective logic (ownership, packing, averaging reduce-scatter, owner
step, all-gather, unpack) must give every rank the bank that one process
gets by stepping every matrix on the mean gradient. The local step here is
the oracle, so the comparison is exact; the library's own step is covered by
the GPU parity tests.
"""
import dataclasses
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from muon_newton_schulz_05_b200.sharded import ShardPlan, ns_work  # noqa: E402

SHAPES = [(3, 16, 24), (2, 40, 8), (1, 8, 8)]
GPT_SHAPES = [(48, 768, 768), (12, 768, 3072), (12, 3072, 768)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _hp_dict(hp):
    d = dataclasses.asdict(hp)
    d["coeffs"] = [tuple(c) for c in d["coeffs"]]
    return d


def _oracle_step_fn(variant):
    """A local step with the library's signature, computed by the oracle."""
    from oracle import muon_oracle as oracle

    def step(banks, hp, workspace):
        h = _hp_dict(hp)
        for bk in banks:
            dt = "bf16" if bk.param.dtype == torch.bfloat16 else "f32"
            for i in range(bk.param.shape[0]):
                th = bk.param[i].double().numpy()
                g = bk.grad[i].double().numpy()
                if variant == "anvil":
                    t1, mf, ms, _, _ = oracle.anvil_step(th, g, bk.momentum[i].double().numpy(),
                                                         bk.momentum_slow[i].double().numpy(), h, dt)
                    bk.momentum_slow[i] = torch.from_numpy(ms).float()
                    bk.momentum[i] = torch.from_numpy(mf).float()
                else:
                    t1, m1, _ = oracle.muon_step(th, g, bk.momentum[i].double().numpy(), h, dt)
                    bk.momentum[i] = torch.from_numpy(m1).float()
                bk.param[i] = torch.from_numpy(t1).to(bk.param.dtype)
                if bk.ema is not None:
                    e = oracle.ema_update(bk.ema[i].double().numpy(), bk.param[i].double().numpy(),
                                          hp.ema_beta)
                    bk.ema[i] = torch.from_numpy(e).float()
    return step


def _hparams(variant):
    from muon_newton_schulz_05_b200 import Hparams
    if variant == "anvil":
        return Hparams(lr=0.05, weight_decay=0.1, coeffs=[(3.4445, -4.7750, 2.0315)] * 6,
                       beta_fast=0.9, beta_slow=0.99, ema_beta=0.9)
    return Hparams(lr=0.05, mu=0.95, weight_decay=0.01, nesterov=True)


def _params(shapes):
    g = torch.Generator().manual_seed(7)
    return [torch.randn(c, r, k, generator=g).to(torch.bfloat16) for c, r, k in shapes]


def _grads(shapes, rank, step):
    g = torch.Generator().manual_seed(1000 * step + rank + 1)
    return [torch.randn(c, r, k, generator=g) * (1 + rank) for c, r, k in shapes]


def _rank_main(rank, world, port, variant, buckets, steps, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from muon_newton_schulz_05_b200.sharded import ShardedMuon
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        opt = ShardedMuon(SHAPES, torch.bfloat16, torch.float32, variant=variant,
                          buckets=buckets, ema=(variant == "anvil"),
                          step_fn=_oracle_step_fn(variant), workspace_fn=lambda shapes: None)
        params = _params(SHAPES)
        hp = _hparams(variant)
        for s in range(steps):
            opt.step(params, _grads(SHAPES, rank, s), hp)
        res = {"params": [p.float().numpy() for p in params]}
        if variant == "anvil":
            ema = [torch.zeros(c, r, k) for c, r, k in SHAPES]
            opt.gather_ema(ema)
            res["ema"] = [e.numpy() for e in ema]
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _single_process(variant, steps, world):
    """Every matrix stepped by one process on the mean of the ranks' gradients."""
    from muon_newton_schulz_05_b200 import Bank
    params = _params(SHAPES)
    mom = [torch.zeros(c, r, k) for c, r, k in SHAPES]
    slow = [torch.zeros(c, r, k) for c, r, k in SHAPES] if variant == "anvil" else [None] * 3
    ema = [p.float().clone() for p in params] if variant == "anvil" else [None] * 3
    step = _oracle_step_fn(variant)
    hp = _hparams(variant)
    for s in range(steps):
        gs = [_grads(SHAPES, r, s) for r in range(world)]
        mean = [(gs[0][b] + gs[1][b]) / world for b in range(len(SHAPES))]
        step([Bank(params[b], mean[b], mom[b], slow[b], ema[b]) for b in range(len(SHAPES))],
             hp, None)
    return params, ema


def _run(variant, buckets, steps=2, world=2):
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, variant, buckets, steps, out), nprocs=world,
                 join=True)
        return dict(out)


@pytest.mark.parametrize("variant,buckets", [("muon", None), ("muon", [[0], [1, 2]]),
                                             ("anvil", [[2], [0, 1]])])
def test_sharded_step_equals_single_process_step(variant, buckets):
    res = _run(variant, buckets)
    ref_params, ref_ema = _single_process(variant, 2, 2)
    for b in range(len(SHAPES)):
        want = ref_params[b].float().numpy()
        for r in (0, 1):
            np.testing.assert_array_equal(res[r]["params"][b], want)
        if variant == "anvil":
            for r in (0, 1):
                np.testing.assert_array_equal(res[r]["ema"][b], ref_ema[b].numpy())
    # the step moved every matrix
    p0 = _params(SHAPES)
    for b in range(len(SHAPES)):
        assert np.all(np.abs(res[0]["params"][b] - p0[b].float().numpy()).reshape(
            SHAPES[b][0], -1).max(axis=1) > 0)


def _int_grads(shapes, rank, step):
    """Integer-valued gradients: their sums over ranks are exact in any order."""
    g = torch.Generator().manual_seed(77 * step + rank + 5)
    return [torch.randint(-8, 9, (c, r, k), generator=g).float() for c, r, k in shapes]


def _three_rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from muon_newton_schulz_05_b200.sharded import ShardedMuon
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        opt = ShardedMuon(SHAPES, torch.bfloat16, torch.float32, buckets=[[2], [0, 1]],
                          step_fn=_oracle_step_fn("muon"), workspace_fn=lambda shapes: None)
        owns = [len(o) for bk in opt.plan.buckets for o in bk.owned[rank]]
        params = _params(SHAPES)
        for s in range(2):
            opt.step(params, _int_grads(SHAPES, rank, s), _hparams("muon"))
        out[rank] = ([p.float().numpy() for p in params], owns)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_three_ranks_with_ranks_that_own_nothing_in_a_bucket():
    """Bucket [bank 2] has one matrix: two of three ranks send and receive only
    padding there. Every rank still ends with the single-process result."""
    world, port = 3, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_three_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert sum(1 for r in range(world) if res[r][1][0] == 0) == 2   # bucket 0: one owner
    from muon_newton_schulz_05_b200 import Bank
    params = _params(SHAPES)
    mom = [torch.zeros(c, r, k) for c, r, k in SHAPES]
    step = _oracle_step_fn("muon")
    for s in range(2):
        gs = [_int_grads(SHAPES, r, s) for r in range(world)]
        mean = [(gs[0][b] + gs[1][b] + gs[2][b]) / world for b in range(len(SHAPES))]
        step([Bank(params[b], mean[b], mom[b]) for b in range(len(SHAPES))], _hparams("muon"), None)
    for r in range(world):
        for b in range(len(SHAPES)):
            np.testing.assert_array_equal(res[r][0][b], params[b].float().numpy())


def _split_rank(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from muon_newton_schulz_05_b200.sharded import ShardedMuon
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        def make():
            return ShardedMuon(SHAPES, torch.bfloat16, torch.float32, buckets=[[0], [1], [2]],
                               step_fn=_oracle_step_fn("muon"), workspace_fn=lambda shapes: None)
        hp = _hparams("muon")
        a, pa = make(), _params(SHAPES)
        b, pb = make(), _params(SHAPES)
        for s in range(2):
            g = _grads(SHAPES, rank, s)
            a.step(pa, g, hp)
            for k in (2, 1, 0):        # the backward pass finishes the last bucket first
                b.grad_ready(k, g)
            b.finish(pb, hp)
        same = all(torch.equal(x, y) for x, y in zip(pa, pb))
        errors = []
        try:
            b.finish(pb, hp)            # no bucket is ready
        except RuntimeError:
            errors.append("finish")
        b.grad_ready(0, _grads(SHAPES, rank, 9))
        try:
            b.grad_ready(0, _grads(SHAPES, rank, 9))
        except RuntimeError:
            errors.append("twice")
        out[rank] = (same, errors)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_grad_ready_then_finish_equals_step():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_split_rank, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    for r in (0, 1):
        assert res[r] == (True, ["finish", "twice"]), res


def _resume_rank(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from muon_newton_schulz_05_b200.sharded import ShardedMuon
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        def make():
            return ShardedMuon(SHAPES, torch.bfloat16, torch.float32, variant="anvil",
                               buckets=[[2], [0, 1]], ema=True,
                               step_fn=_oracle_step_fn("anvil"), workspace_fn=lambda shapes: None)
        hp = _hparams("anvil")
        straight, params_a = make(), _params(SHAPES)
        for s in range(4):
            straight.step(params_a, _grads(SHAPES, rank, s), hp)
        first, params_b = make(), _params(SHAPES)
        for s in range(2):
            first.step(params_b, _grads(SHAPES, rank, s), hp)
        saved = first.state_dict()
        resumed = make()              # a fresh optimizer, as after a restart
        resumed.load_state_dict(saved)
        for s in range(2, 4):
            resumed.step(params_b, _grads(SHAPES, rank, s), hp)
        same = all(torch.equal(a, b) for a, b in zip(params_a, params_b))
        ema_a = [torch.zeros(c, r, k) for c, r, k in SHAPES]
        ema_b = [torch.zeros(c, r, k) for c, r, k in SHAPES]
        straight.gather_ema(ema_a)
        resumed.gather_ema(ema_b)
        same_ema = all(torch.equal(a, b) for a, b in zip(ema_a, ema_b))
        wrong = ShardedMuon(SHAPES, torch.bfloat16, torch.float32, variant="anvil", ema=True,
                            step_fn=_oracle_step_fn("anvil"), workspace_fn=lambda shapes: None)
        try:
            wrong.load_state_dict(saved)   # one bucket instead of two: another plan
            rejected = False
        except ValueError:
            rejected = True
        out[rank] = (same, same_ema, rejected)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_sharded_state_resumes_bitwise():
    """2 steps, save each rank's shard state, a fresh optimizer loads it, 2
    more steps: the same bank and EMA as 4 steps straight."""
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_resume_rank, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == (True, True, True) and res[1] == (True, True, True), res


def test_plan_owns_every_matrix_once_and_balances_gpt_bank():
    for world in (1, 2, 4, 8):
        for buckets in (None, [[0, 1, 2]]):   # default: one bucket per bank
            plan = ShardPlan.build(GPT_SHAPES, world, buckets)
            if buckets is None:
                assert [bk.banks for bk in plan.buckets] == [[0], [1], [2]]
            for b, (count, rows, cols) in enumerate(GPT_SHAPES):
                k, j = next((k, j) for k, bk in enumerate(plan.buckets)
                            for j, x in enumerate(bk.banks) if x == b)
                got = sorted(i for r in range(world) for i in plan.buckets[k].owned[r][j])
                assert got == list(range(count))
        plan = ShardPlan.build(GPT_SHAPES, world, [[0, 1, 2]])
        total = sum(c * ns_work(r, k) for c, r, k in GPT_SHAPES)
        assert abs(sum(plan.load) - total) < 1e-6 * total
        # 72 matrices of two weights: greedy lands within one small matrix of even
        assert max(plan.load) - total / world <= ns_work(768, 768) + 1e-6 * total


def test_plan_segments_aligned_and_pack_roundtrip():
    plan = ShardPlan.build(SHAPES, 3, [[1], [0, 2]])
    ts = [torch.arange(c * r * k, dtype=torch.float32).view(c, r, k) + 1000 * i
          for i, (c, r, k) in enumerate(SHAPES)]
    for k, bk in enumerate(plan.buckets):
        for r in range(3):
            assert all(o % 128 == 0 for o in bk.offsets[r])
            used = [len(o) * SHAPES[b][1] * SHAPES[b][2] for o, b in zip(bk.owned[r], bk.banks)]
            assert bk.offsets[r][-1] + used[-1] <= bk.seg
        flat = torch.full((3 * bk.seg,), -1.0)
        plan.pack(k, ts, flat)
        back = [torch.zeros_like(t) for t in ts]
        plan.unpack(k, flat, back)
        for b in bk.banks:
            assert torch.equal(back[b], ts[b])


def test_plan_rejects_bad_buckets():
    with pytest.raises(ValueError):
        ShardPlan.build(SHAPES, 2, [[0], [1]])
    with pytest.raises(ValueError):
        ShardPlan.build(SHAPES, 2, [[0, 1], [1, 2]])
    with pytest.raises(ValueError):
        ShardPlan.build(SHAPES, 0)


# ---------------------------------------------------------------------------
# Owner-ordered bank storage (ShardedBankMuon): no packing copies
# ---------------------------------------------------------------------------
from muon_newton_schulz_05_b200.sharded import OwnerLayout  # noqa: E402


def _bank_rank_main(rank, world, port, variant, steps, order, out, per_bank=False):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from muon_newton_schulz_05_b200.sharded import ShardedBankMuon
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        opt = ShardedBankMuon(SHAPES, torch.bfloat16, torch.float32, variant=variant,
                              ema=(variant == "anvil"), step_fn=_oracle_step_fn(variant),
                              workspace_fn=lambda shapes: None, per_bank=per_bank)
        for p, p0 in zip(opt.params, _params(SHAPES)):
            p.copy_(p0)
        hp = _hparams(variant)
        for s in range(steps):
            for g, g0 in zip(opt.grads, _grads(SHAPES, rank, s)):
                g.copy_(g0)
            for b in order:            # the order the backward pass finishes the banks
                opt.grad_ready(b)
            opt.finish(hp)
        res = {"params": [p.float().numpy().copy() for p in opt.params],
               "owned": list(opt.owned)}
        if variant == "anvil":
            ema = [torch.zeros(c, r, k) for c, r, k in SHAPES]
            opt.gather_ema(ema)
            res["ema"] = [e.numpy() for e in ema]
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("variant,world,order,per_bank",
                         [("muon", 2, [0, 1, 2], False), ("anvil", 2, [2, 1, 0], True),
                          ("muon", 3, [1, 0, 2], False), ("muon", 2, [1, 2, 0], True)])
def test_bank_storage_step_equals_single_process_step(variant, world, order, per_bank):
    """Every rank ends with the bank one process gets by stepping every matrix
    on the mean of the ranks' gradients (gradients summed in the same order on
    both sides for two ranks; three ranks use integer-exact sums below)."""
    port = _free_port()
    steps = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_bank_rank_main, args=(world, port, variant, steps, order, out, per_bank),
                 nprocs=world, join=True)
        res = dict(out)
    # every matrix owned by exactly one rank
    for b, (count, _, _) in enumerate(SHAPES):
        got = sorted(i for r in range(world) for i in range(*res[r]["owned"][b]))
        assert got == list(range(count))
    if world == 2:
        ref_params, ref_ema = _single_process(variant, steps, world)
        for b in range(len(SHAPES)):
            for r in range(world):
                np.testing.assert_array_equal(res[r]["params"][b], ref_params[b].float().numpy())
                if variant == "anvil":
                    np.testing.assert_array_equal(res[r]["ema"][b], ref_ema[b].numpy())
    else:
        # float sums over three ranks may round differently: every rank agrees,
        # and each matches the single-process step closely
        from muon_newton_schulz_05_b200 import Bank
        params = _params(SHAPES)
        mom = [torch.zeros(c, r, k) for c, r, k in SHAPES]
        step = _oracle_step_fn("muon")
        for s in range(steps):
            gs = [_grads(SHAPES, r, s) for r in range(world)]
            mean = [sum(g[b] for g in gs) / world for b in range(len(SHAPES))]
            step([Bank(params[b], mean[b], mom[b]) for b in range(len(SHAPES))], _hparams("muon"), None)
        for b in range(len(SHAPES)):
            for r in range(1, world):
                np.testing.assert_array_equal(res[r]["params"][b], res[0]["params"][b])
            np.testing.assert_allclose(res[0]["params"][b], params[b].float().numpy(),
                                       rtol=0, atol=2e-2 * np.abs(params[b].float().numpy()).max())


def test_owner_layout_covers_every_matrix_and_balances():
    for world in (1, 2, 3, 4, 8):
        lay = OwnerLayout.build(GPT_SHAPES, world)
        total = sum(c * ns_work(r, k) for c, r, k in GPT_SHAPES)
        assert abs(sum(lay.load) - total) < 1e-6 * total
        for (count, _, _), sl in zip(GPT_SHAPES, lay.banks):
            runs = [sl.owned(r) for r in range(world)]
            assert [i for lo, hi in runs for i in range(lo, hi)] == list(range(count))
            assert sl.offset + count <= world * sl.seg and sl.seg == -(-count // world)
        # divisible counts split evenly; 12 large matrices over 8 ranks cannot
        if world in (1, 2, 3, 4):
            assert max(lay.load) == pytest.approx(total / world, rel=1e-12)
        else:
            assert max(lay.load) <= 1.25 * total / world
    with pytest.raises(ValueError):
        OwnerLayout.build(GPT_SHAPES, 0)


def _bank_resume_rank(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from muon_newton_schulz_05_b200.sharded import ShardedBankMuon
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        def make():
            o = ShardedBankMuon(SHAPES, torch.bfloat16, torch.float32, variant="anvil", ema=True,
                                step_fn=_oracle_step_fn("anvil"), workspace_fn=lambda shapes: None)
            for p, p0 in zip(o.params, _params(SHAPES)):
                p.copy_(p0)
            return o
        hp = _hparams("anvil")

        def run(o, steps):
            for s in steps:
                for g, g0 in zip(o.grads, _grads(SHAPES, rank, s)):
                    g.copy_(g0)
                o.step(hp)
        a = make()
        run(a, range(4))
        b = make()
        run(b, range(2))
        saved = b.state_dict()
        c = make()
        for p, q in zip(c.params, b.params):   # the weights come from the model checkpoint
            p.copy_(q)
        c.load_state_dict(saved)
        run(c, range(2, 4))
        same = all(torch.equal(x, y) for x, y in zip(a.params, c.params))
        ea = [torch.zeros(cc, r, k) for cc, r, k in SHAPES]
        ec = [torch.zeros(cc, r, k) for cc, r, k in SHAPES]
        a.gather_ema(ea)
        c.gather_ema(ec)
        out[rank] = (same, all(torch.equal(x, y) for x, y in zip(ea, ec)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_bank_storage_state_resumes_bitwise():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_bank_resume_rank, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == (True, True) and res[1] == (True, True), res

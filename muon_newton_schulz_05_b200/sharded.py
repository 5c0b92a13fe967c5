"""Data-parallel Muon over a process group: each matrix has one owner rank.

In data-parallel training every rank holds the whole bank and its own
gradient. Muon's matrix products can be spread over the GPUs layer by layer
(page "きみはNanoGPT speedrunを知っているか？", section "おまけ"). Here every
matrix gets one owner, chosen so that the ranks' Newton-Schulz flops
(3 r^2 c + r^3 per iteration, r <= c the short side) come out balanced:
largest first, each to the least-loaded rank. One step, per bucket of banks:

  1. reduce-scatter: gradients packed in owner order are averaged over the
     ranks; each rank receives the gradients of the matrices it owns;
  2. the owner runs the optimizer step (the CUDA library) on its matrices
     only, so momentum and workspace live on one rank;
  3. all-gather: the owners' updated parameters reach every rank, which
     unpacks them into its bank.

`step` issues all reduce-scatters at once (asynchronous); bucket k's step
waits only for bucket k's, so on NCCL the exchange of later buckets overlaps
the Newton-Schulz chain of earlier ones, and each bucket's all-gather
overlaps the next bucket's step. A training loop can start each bucket's
exchange as soon as the backward pass has finished its gradients
(`grad_ready(k, grads)`, every rank in the same order) and call `finish`
after the last one. The packing and unpacking are plain copies; every
arithmetic step of the optimizer runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence, Tuple

# every bank's slot in a segment starts on a 256-byte boundary (the library
# wants 16-byte aligned operands; 256 also keeps NCCL on its vector path)
_ALIGN_ELEMS = 128


def ns_work(rows: int, cols: int) -> float:
    """Newton-Schulz flops of one iteration on a rows x cols matrix, over 2."""
    r, c = min(rows, cols), max(rows, cols)
    return 3.0 * r * r * c + float(r) ** 3


def _round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


@dataclass
class Bucket:
    banks: List[int]                 # bank indices in this bucket
    owned: List[List[List[int]]]     # owned[rank][j] = matrix indices of banks[j]
    offsets: List[List[int]]         # offsets[rank][j] = element offset in the segment
    seg: int                         # elements per rank segment (padded)


@dataclass
class ShardPlan:
    world: int
    shapes: List[Tuple[int, int, int]]
    owner: List[List[int]]           # owner[b][i]
    buckets: List[Bucket]
    load: List[float]                # per-rank Newton-Schulz work

    @classmethod
    def build(cls, shapes: Sequence[Tuple[int, int, int]], world: int,
              buckets: Optional[Sequence[Sequence[int]]] = None) -> "ShardPlan":
        """buckets: lists of bank indices (default: one bucket per bank, so the
        exchange of later banks overlaps the step of earlier ones).
        Owners are assigned bucket by bucket with the load carried over, so
        each bucket and the whole step are both close to balanced."""
        shapes = [tuple(int(v) for v in s) for s in shapes]
        if world < 1:
            raise ValueError("world size must be >= 1")
        groups = [list(g) for g in buckets] if buckets is not None else [[b] for b in range(len(shapes))]
        seen = sorted(b for g in groups for b in g)
        if seen != list(range(len(shapes))):
            raise ValueError("buckets must list every bank exactly once")
        load = [0.0] * world
        owner = [[0] * s[0] for s in shapes]
        out = []
        for g in groups:
            items = sorted(((-ns_work(shapes[b][1], shapes[b][2]), b, i)
                            for b in g for i in range(shapes[b][0])))
            for negw, b, i in items:
                r = min(range(world), key=lambda k: (load[k], k))
                owner[b][i] = r
                load[r] -= negw
            owned = [[[i for i in range(shapes[b][0]) if owner[b][i] == r] for b in g]
                     for r in range(world)]
            offsets, seg = [], 0
            for r in range(world):
                pos, offs = 0, []
                for j, b in enumerate(g):
                    offs.append(pos)
                    pos += _round_up(len(owned[r][j]) * shapes[b][1] * shapes[b][2], _ALIGN_ELEMS)
                offsets.append(offs)
                seg = max(seg, pos)
            out.append(Bucket(g, owned, offsets, max(seg, _ALIGN_ELEMS)))
        return cls(world, list(shapes), owner, out, load)

    def views(self, k: int, rank: int, seg_flat) -> List:
        """[n_owned, R, C] views of rank's segment of bucket k, one per bank of
        the bucket (None where the rank owns no matrix of that bank)."""
        bk = self.buckets[k]
        out = []
        for j, b in enumerate(bk.banks):
            n = len(bk.owned[rank][j])
            _, rows, cols = self.shapes[b]
            o = bk.offsets[rank][j]
            out.append(seg_flat[o:o + n * rows * cols].view(n, rows, cols) if n else None)
        return out

    def pack(self, k: int, tensors: Sequence, flat) -> None:
        """Bank tensors -> flat (world * seg of bucket k), segment r holding
        rank r's matrices. Padding is left as it is."""
        seg = self.buckets[k].seg
        for r in range(self.world):
            for j, v in enumerate(self.views(k, r, flat[r * seg:(r + 1) * seg])):
                if v is not None:
                    v.copy_(tensors[self.buckets[k].banks[j]][self.buckets[k].owned[r][j]])

    def unpack(self, k: int, flat, tensors: Sequence) -> None:
        """Inverse of pack for bucket k."""
        seg = self.buckets[k].seg
        for r in range(self.world):
            for j, v in enumerate(self.views(k, r, flat[r * seg:(r + 1) * seg])):
                if v is not None:
                    tensors[self.buckets[k].banks[j]][self.buckets[k].owned[r][j]] = v


class ShardedMuon:
    """Owner-sharded data-parallel Muon (or ANVIL) step for a list of banks.

    params: this rank's full bank tensors [count, R, C], identical on every
    rank and overwritten with the updated bank; grads: this rank's local
    gradients of the same shapes. Each rank keeps fp32 momentum (ANVIL: both
    momenta, and the EMA when ema=True) for the matrices it owns only.
    step_fn(banks, hp, workspace) runs the local step on Bank objects and
    defaults to the library's muon_step (anvil_step for variant="anvil");
    workspace_fn(shapes) allocates its workspace.
    """

    def __init__(self, shapes, param_dtype, grad_dtype, group=None, variant: str = "muon",
                 device=None, buckets=None, ema: bool = False,
                 step_fn: Optional[Callable] = None, workspace_fn: Optional[Callable] = None):
        import torch
        import torch.distributed as dist
        if variant not in ("muon", "anvil"):
            raise ValueError("variant must be 'muon' or 'anvil'")
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.gloo = dist.get_backend(group) == "gloo"
        self.plan = ShardPlan.build(shapes, self.world, buckets)
        self.variant = variant
        self.device = device if device is not None else torch.device("cpu")
        if step_fn is None or workspace_fn is None:
            from . import alloc_workspace, anvil_step, muon_step
            step_fn = step_fn or (anvil_step if variant == "anvil" else muon_step)
            workspace_fn = workspace_fn or (lambda shapes: alloc_workspace(shapes, self.device))
        self.step_fn, self.workspace_fn = step_fn, workspace_fn
        self.workspaces: List = [None] * len(self.plan.buckets)
        self._gflat, self._gseg, self._pflat, self._pseg = [], [], [], []
        self.momentum, self.momentum_slow, self.ema = [], [], []
        for k, bk in enumerate(self.plan.buckets):
            n = self.world * bk.seg
            self._gflat.append(torch.zeros(n, dtype=grad_dtype, device=self.device))
            self._gseg.append(torch.zeros(bk.seg, dtype=grad_dtype, device=self.device))
            self._pflat.append(torch.zeros(n, dtype=param_dtype, device=self.device))
            self._pseg.append(torch.zeros(bk.seg, dtype=param_dtype, device=self.device))

            def state(on):
                return [torch.zeros(len(o), *self.plan.shapes[b][1:], dtype=torch.float32,
                                    device=self.device) if (o and on) else None
                        for o, b in zip(bk.owned[self.rank], bk.banks)]
            self.momentum.append(state(True))
            self.momentum_slow.append(state(variant == "anvil"))
            self.ema.append(state(ema))
        self._ema_ready = False
        self._pending: List = [None] * len(self.plan.buckets)   # reduce-scatters in flight

    def plan_signature(self) -> Tuple:
        """What a saved state depends on: world size, bank shapes, buckets and
        the resulting ownership."""
        return (self.world, tuple(self.plan.shapes),
                tuple(tuple(bk.banks) for bk in self.plan.buckets),
                tuple(tuple(o) for o in self.plan.owner))

    def state_dict(self) -> dict:
        """This rank's optimizer state (its owned matrices' momenta and EMA),
        as CPU tensors, with the plan it belongs to. Save one per rank."""
        def cpu(lists):
            return [[t.detach().cpu().clone() if t is not None else None for t in ts] for ts in lists]
        return {"plan": self.plan_signature(), "rank": self.rank, "variant": self.variant,
                "momentum": cpu(self.momentum), "momentum_slow": cpu(self.momentum_slow),
                "ema": cpu(self.ema), "ema_ready": self._ema_ready}

    def load_state_dict(self, state: dict) -> None:
        """Restore a state saved by the same rank under the same plan."""
        if state["plan"] != self.plan_signature() or state["rank"] != self.rank:
            raise ValueError("the state was saved under another ownership plan or rank")
        if state["variant"] != self.variant:
            raise ValueError("the state was saved by the other variant")
        for name in ("momentum", "momentum_slow", "ema"):
            mine, saved = getattr(self, name), state[name]
            for ts, ss in zip(mine, saved):
                for t, v in zip(ts, ss):
                    if (t is None) != (v is None):
                        raise ValueError(f"{name}: the saved state has a different layout")
                    if t is not None:
                        t.copy_(v)
        self._ema_ready = bool(state["ema_ready"])

    def owned_shapes(self, k: int) -> List[Tuple[int, int, int]]:
        bk = self.plan.buckets[k]
        return [(len(o), *self.plan.shapes[b][1:]) for o, b in zip(bk.owned[self.rank], bk.banks) if o]

    def _reduce_scatter(self, k: int):
        """Start bucket k's averaging reduce-scatter: its work handle, or True
        when it is already complete (gloo)."""
        if self.gloo:
            # gloo has no reduce-scatter: sum everywhere, keep this rank's segment
            self.dist.all_reduce(self._gflat[k], op=self.dist.ReduceOp.SUM, group=self.group)
            seg = self.plan.buckets[k].seg
            self._gseg[k].copy_(self._gflat[k][self.rank * seg:(self.rank + 1) * seg])
            self._gseg[k].div_(self.world)
            return True
        return self.dist.reduce_scatter_tensor(self._gseg[k], self._gflat[k],
                                               op=self.dist.ReduceOp.AVG, group=self.group,
                                               async_op=True)

    def _all_gather(self, k: int):
        if self.gloo:
            self.dist.all_gather(list(self._pflat[k].chunk(self.world)), self._pseg[k],
                                 group=self.group)
            return None
        return self.dist.all_gather_into_tensor(self._pflat[k], self._pseg[k],
                                                group=self.group, async_op=True)

    def grad_ready(self, k: int, grads: Sequence) -> None:
        """Bucket k's gradients are final (grads: this rank's bank tensors, only
        bucket k's banks are read): pack them and start their averaging
        reduce-scatter now, so the exchange overlaps the rest of the backward
        pass. Each bucket once per step, in any order that is the same on every
        rank (collectives must match), then `finish`."""
        if self._pending[k] is not None:
            raise RuntimeError(f"bucket {k} is already in flight in this step")
        self.plan.pack(k, grads, self._gflat[k])
        self._pending[k] = self._reduce_scatter(k)

    def finish(self, params: Sequence, hp) -> None:
        """Step every bucket whose reduce-scatter `grad_ready` started (all must
        have been), in bucket order, and bring the updated parameters to
        every rank."""
        from . import Bank
        plan, rank = self.plan, self.rank
        if any(w is None for w in self._pending):
            raise RuntimeError("every bucket needs grad_ready before finish")
        ag = []
        for k, bk in enumerate(plan.buckets):
            if self._pending[k] is not True:
                self._pending[k].wait()
            gv = plan.views(k, rank, self._gseg[k])
            pv = plan.views(k, rank, self._pseg[k])
            banks = []
            for j, b in enumerate(bk.banks):
                if pv[j] is None:
                    continue
                pv[j].copy_(params[b][bk.owned[rank][j]])
                banks.append(Bank(pv[j], gv[j], self.momentum[k][j], self.momentum_slow[k][j],
                                  self.ema[k][j]))
            if banks:
                if self.workspaces[k] is None:
                    self.workspaces[k] = self.workspace_fn([bank.shape for bank in banks])
                if any(e is not None for e in self.ema[k]):
                    self._init_ema(k, pv)
                self.step_fn(banks, hp, self.workspaces[k])
            ag.append(self._all_gather(k))
        for k in range(len(plan.buckets)):
            if ag[k] is not None:
                ag[k].wait()
            plan.unpack(k, self._pflat[k], params)
        self._pending = [None] * len(plan.buckets)
        self._ema_ready = True

    def step(self, params: Sequence, grads: Sequence, hp) -> None:
        """One data-parallel step: every bucket's exchange, then `finish`."""
        for k in range(len(self.plan.buckets)):
            self.grad_ready(k, grads)
        self.finish(params, hp)

    def _init_ema(self, k: int, pv) -> None:
        # the average starts at the parameters it averages
        if self._ema_ready:
            return
        for e, p in zip(self.ema[k], pv):
            if e is not None:
                e.copy_(p)

    def gather_ema(self, out: Sequence) -> None:
        """Collect the owners' EMA of every matrix into out (fp32 bank tensors)."""
        import torch
        for k, bk in enumerate(self.plan.buckets):
            seg = torch.zeros(bk.seg, dtype=torch.float32, device=self.device)
            for v, e in zip(self.plan.views(k, self.rank, seg), self.ema[k]):
                if v is not None:
                    if e is None:
                        raise RuntimeError("ShardedMuon was built without ema=True")
                    v.copy_(e)
            flat = torch.zeros(self.world * bk.seg, dtype=torch.float32, device=self.device)
            if self.gloo:
                self.dist.all_gather(list(flat.chunk(self.world)), seg, group=self.group)
            else:
                self.dist.all_gather_into_tensor(flat, seg, group=self.group)
            self.plan.unpack(k, flat, out)


# ---------------------------------------------------------------------------
# Owner-ordered bank storage: the same step without any packing copies
# ---------------------------------------------------------------------------
@dataclass
class BankSlots:
    """Where one bank lives in its owner-ordered buffer. The buffer holds
    world * seg matrix slots; rank r owns slots [r seg, (r + 1) seg); the
    bank's count matrices fill slots [offset, offset + count) in order, the
    rest is padding."""
    count: int
    seg: int
    offset: int

    def owned(self, rank: int) -> Tuple[int, int]:
        """Matrices [lo, hi) of the bank that rank owns (lo == hi: none)."""
        lo = max(rank * self.seg, self.offset) - self.offset
        hi = min((rank + 1) * self.seg, self.offset + self.count) - self.offset
        return lo, max(lo, hi)


@dataclass
class OwnerLayout:
    world: int
    shapes: List[Tuple[int, int, int]]
    banks: List[BankSlots]
    load: List[float]                # per-rank Newton-Schulz work

    @classmethod
    def build(cls, shapes: Sequence[Tuple[int, int, int]], world: int) -> "OwnerLayout":
        """Each bank gets ceil(count / world) slots per rank, so every rank owns
        a contiguous run of its matrices; the bank's offset in the buffer (how
        many padding slots come first) is chosen, heaviest banks first, to
        keep the ranks' Newton-Schulz work (3 r^2 c + r^3 per matrix) as even
        as the contiguous runs allow."""
        shapes = [tuple(int(v) for v in s) for s in shapes]
        if world < 1:
            raise ValueError("world size must be >= 1")
        load = [0.0] * world
        slots: List[Optional[BankSlots]] = [None] * len(shapes)
        order = sorted(range(len(shapes)), key=lambda b: (-ns_work(shapes[b][1], shapes[b][2]), b))
        for b in order:
            count, rows, cols = shapes[b]
            seg = -(-count // world)
            w = ns_work(rows, cols)
            best = None
            for off in range(world * seg - count + 1):
                cand = BankSlots(count, seg, off)
                new = [load[r] + w * (lambda lh: lh[1] - lh[0])(cand.owned(r)) for r in range(world)]
                key = (max(new), sum(x * x for x in new), off)
                if best is None or key < best[0]:
                    best = (key, cand, new)
            slots[b] = best[1]
            load = best[2]
        return cls(world, shapes, slots, load)

    def signature(self) -> Tuple:
        return (self.world, tuple(self.shapes),
                tuple((s.count, s.seg, s.offset) for s in self.banks))


class ShardedBankMuon:
    """Owner-sharded data-parallel Muon (or ANVIL) step on bank storage that the
    optimizer owns, laid out in owner order (see OwnerLayout): no gradient is
    packed and no parameter is unpacked.

    `params[b]` and `grads[b]` are this rank's [count, R, C] bank tensors,
    views into one flat buffer per bank: load the model's weights into
    `params` (identical on every rank) and let the backward pass write this
    rank's gradients into `grads`. One step: an averaging reduce-scatter of
    every bank's gradient buffer in place (each rank receives its own slots);
    the optimizer step (the CUDA library, one call over all banks) on the
    matrices this rank owns, in place; an all-gather of every parameter
    buffer in place. Momenta (and the EMA) exist only for the owned matrices.
    A training loop may call `grad_ready(b)` as soon as bank b's gradients
    are final, then `finish(hp)`; `step(hp)` does both.
    per_bank=False (default) steps every bank's owned matrices in one library
    call (one Newton-Schulz chain over all of them: the most work per launch).
    per_bank=True steps each bank as soon as its reduce-scatter has landed and
    starts that bank's all-gather right after, so on NCCL the exchange of
    later banks overlaps the chains of earlier ones.
    Requires rows * cols to be a multiple of 8, so that every matrix slot
    starts on a 16-byte boundary.
    """

    def __init__(self, shapes, param_dtype, grad_dtype, group=None, variant: str = "muon",
                 device=None, ema: bool = False, step_fn: Optional[Callable] = None,
                 workspace_fn: Optional[Callable] = None, per_bank: bool = False):
        import torch
        import torch.distributed as dist
        if variant not in ("muon", "anvil"):
            raise ValueError("variant must be 'muon' or 'anvil'")
        shapes = [tuple(int(v) for v in s) for s in shapes]
        for c, r, k in shapes:
            if (r * k) % 8:
                raise ValueError(f"rows * cols of a {r} x {k} matrix is not a multiple of 8")
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.gloo = dist.get_backend(group) == "gloo"
        self.layout = OwnerLayout.build(shapes, self.world)
        self.variant = variant
        self.device = device if device is not None else torch.device("cpu")
        if step_fn is None or workspace_fn is None:
            from . import alloc_workspace, anvil_step, muon_step
            step_fn = step_fn or (anvil_step if variant == "anvil" else muon_step)
            workspace_fn = workspace_fn or (lambda shapes: alloc_workspace(shapes, self.device))
        self.step_fn, self.workspace_fn = step_fn, workspace_fn
        self._pflat, self._gflat = [], []
        self.params, self.grads = [], []
        self.momentum, self.momentum_slow, self.ema = [], [], []
        self.owned = []
        for (count, rows, cols), sl in zip(shapes, self.layout.banks):
            rc = rows * cols
            n = self.world * sl.seg * rc
            pf = torch.zeros(n, dtype=param_dtype, device=self.device)
            gf = torch.zeros(n, dtype=grad_dtype, device=self.device)
            self._pflat.append(pf)
            self._gflat.append(gf)
            self.params.append(pf[sl.offset * rc:(sl.offset + count) * rc].view(count, rows, cols))
            self.grads.append(gf[sl.offset * rc:(sl.offset + count) * rc].view(count, rows, cols))
            lo, hi = sl.owned(self.rank)
            self.owned.append((lo, hi))

            def state(on):
                if not on or hi == lo:
                    return None
                return torch.zeros(hi - lo, rows, cols, dtype=torch.float32, device=self.device)
            self.momentum.append(state(True))
            self.momentum_slow.append(state(variant == "anvil"))
            self.ema.append(state(ema))
        self.per_bank = bool(per_bank)
        self.workspace = None                      # one call over all banks
        self.workspaces: List = [None] * len(shapes)  # per_bank: one per bank
        self._ema_ready = False
        self._pending: List = [None] * len(shapes)

    def _segment(self, flat, b):
        sl = self.layout.banks[b]
        rc = self.layout.shapes[b][1] * self.layout.shapes[b][2]
        return flat[self.rank * sl.seg * rc:(self.rank + 1) * sl.seg * rc]

    def owned_shapes(self) -> List[Tuple[int, int, int]]:
        return [(hi - lo, s[1], s[2]) for (lo, hi), s in zip(self.owned, self.layout.shapes)
                if hi > lo]

    def grad_ready(self, b: int) -> None:
        """Bank b's gradients in `grads[b]` are final: start their averaging
        reduce-scatter (in place: this rank's slots receive the mean)."""
        if self._pending[b] is not None:
            raise RuntimeError(f"bank {b} is already in flight in this step")
        flat, seg = self._gflat[b], self._segment(self._gflat[b], b)
        if self.gloo:
            # gloo has no reduce-scatter: sum everywhere, scale this rank's slots
            self.dist.all_reduce(flat, op=self.dist.ReduceOp.SUM, group=self.group)
            seg.div_(self.world)
            self._pending[b] = True
        else:
            self._pending[b] = self.dist.reduce_scatter_tensor(
                seg, flat, op=self.dist.ReduceOp.AVG, group=self.group, async_op=True)

    def finish(self, hp) -> None:
        """Step the owned matrices of every bank (all must be grad_ready) with
        one library call, then all-gather every parameter buffer in place."""
        if any(w is None for w in self._pending):
            raise RuntimeError("every bank needs grad_ready before finish")
        nb = len(self.layout.banks)
        works = []
        if self.per_bank:
            for b in range(nb):
                self._wait_rs(b)
                bank = self._owned_bank(b)
                if bank is not None:
                    if self.workspaces[b] is None:
                        self.workspaces[b] = self.workspace_fn([bank.shape])
                    self.step_fn([bank], hp, self.workspaces[b])
                works.append(self._all_gather(b))
        else:
            for b in range(nb):
                self._wait_rs(b)
            banks = [bk for bk in (self._owned_bank(b) for b in range(nb)) if bk is not None]
            if banks:
                if self.workspace is None:
                    self.workspace = self.workspace_fn([bk.shape for bk in banks])
                self.step_fn(banks, hp, self.workspace)
            works = [self._all_gather(b) for b in range(nb)]
        for w in works:
            if w is not None:
                w.wait()
        self._pending = [None] * nb
        self._ema_ready = True

    def _wait_rs(self, b: int) -> None:
        if self._pending[b] is not True:
            self._pending[b].wait()

    def _owned_bank(self, b: int):
        """The library's Bank for this rank's matrices of bank b (None if none)."""
        from . import Bank
        lo, hi = self.owned[b]
        if hi == lo:
            return None
        p, g = self.params[b][lo:hi], self.grads[b][lo:hi]
        if self.ema[b] is not None and not self._ema_ready:
            self.ema[b].copy_(p)  # the average starts at the parameters it averages
        return Bank(p, g, self.momentum[b], self.momentum_slow[b], self.ema[b])

    def _all_gather(self, b: int):
        """Start bank b's in-place all-gather: its work handle (None on gloo,
        where it has completed)."""
        flat, seg = self._pflat[b], self._segment(self._pflat[b], b)
        if self.gloo:
            self.dist.all_gather(list(flat.chunk(self.world)), seg.clone(), group=self.group)
            return None
        return self.dist.all_gather_into_tensor(flat, seg, group=self.group, async_op=True)

    def device_status(self) -> int:
        """Synchronises and returns the first non-zero device status of this
        rank's workspaces (0 when all are clear)."""
        from . import device_status
        for ws in [self.workspace] + list(self.workspaces):
            if ws is not None:
                st = device_status(ws)
                if st:
                    return st
        return 0

    def step(self, hp) -> None:
        for b in range(len(self.layout.banks)):
            self.grad_ready(b)
        self.finish(hp)

    def state_dict(self) -> dict:
        def cpu(ts):
            return [t.detach().cpu().clone() if t is not None else None for t in ts]
        return {"layout": self.layout.signature(), "rank": self.rank, "variant": self.variant,
                "momentum": cpu(self.momentum), "momentum_slow": cpu(self.momentum_slow),
                "ema": cpu(self.ema), "ema_ready": self._ema_ready}

    def load_state_dict(self, state: dict) -> None:
        if state["layout"] != self.layout.signature() or state["rank"] != self.rank:
            raise ValueError("the state was saved under another layout or rank")
        if state["variant"] != self.variant:
            raise ValueError("the state was saved by the other variant")
        for name in ("momentum", "momentum_slow", "ema"):
            for t, v in zip(getattr(self, name), state[name]):
                if (t is None) != (v is None):
                    raise ValueError(f"{name}: the saved state has a different layout")
                if t is not None:
                    t.copy_(v)
        self._ema_ready = bool(state["ema_ready"])

    def gather_ema(self, out: Sequence) -> None:
        """Collect the owners' EMA of every matrix into out (fp32 bank tensors)."""
        import torch
        for b, ((count, rows, cols), sl) in enumerate(zip(self.layout.shapes, self.layout.banks)):
            rc = rows * cols
            flat = torch.zeros(self.world * sl.seg * rc, dtype=torch.float32, device=self.device)
            seg = self._segment(flat, b)
            lo, hi = self.owned[b]
            if hi > lo:
                if self.ema[b] is None:
                    raise RuntimeError("ShardedBankMuon was built without ema=True")
                start = (max(self.rank * sl.seg, sl.offset) - self.rank * sl.seg) * rc
                seg[start:start + (hi - lo) * rc].copy_(self.ema[b].reshape(-1))
            if self.gloo:
                self.dist.all_gather(list(flat.chunk(self.world)), seg.clone(), group=self.group)
            else:
                self.dist.all_gather_into_tensor(flat, seg, group=self.group)
            out[b].copy_(flat[sl.offset * rc:(sl.offset + count) * rc].view(count, rows, cols))

"""Optimizer step overlapped with the backward pass, group by group.

The banks are split into groups (typically by layer, in the order the
backward pass finishes them). As soon as a group's gradients are final,
`grad_ready(i)` makes a side stream wait for that point of the producing
stream and launches the group's step there, so the Newton-Schulz chains of
late layers run while the backward pass of earlier layers is still on the
GPU. `wait()` joins the side stream back. Everything is stream-ordered (no
host synchronisation), so a whole training step, backward pass and
overlapped optimizer included, can be captured in one CUDA graph (the pages
credit whole-step graph capture with seconds of the record: "Training
NanoGPT in 39.9 Seconds", the ablation table's CUDA graphs row).

Call `grad_ready(i)` only after the last use of group i's parameters in the
backward pass: the step writes them in place. The gradients must stay alive
until `wait()` (they are read on the side stream).
"""
from __future__ import annotations

from typing import List, Optional, Sequence


class OverlappedStep:
    """groups: lists of Bank (one library call per group, each with its own
    workspace); variant "muon" or "anvil"; device: the banks' CUDA device."""

    def __init__(self, groups: Sequence[Sequence["object"]], hp, variant: str = "muon",
                 device=None, side_stream=None):
        import torch
        from . import alloc_workspace, anvil_step, muon_step
        if variant not in ("muon", "anvil"):
            raise ValueError("variant must be 'muon' or 'anvil'")
        if not groups or any(len(g) == 0 for g in groups):
            raise ValueError("every group needs at least one bank")
        self.groups: List[list] = [list(g) for g in groups]
        self.hp = hp
        self.step_fn = anvil_step if variant == "anvil" else muon_step
        self.device = device if device is not None else self.groups[0][0].param.device
        self.workspaces = [alloc_workspace([b.shape for b in g], self.device) for g in self.groups]
        self.side = side_stream if side_stream is not None else torch.cuda.Stream(self.device)
        self._ready = [torch.cuda.Event() for _ in self.groups]
        self._done = torch.cuda.Event()
        self._launched = [False] * len(self.groups)

    def grad_ready(self, i: int, stream=None) -> None:
        """Group i's gradients are final on `stream` (default: the current
        stream): launch its step on the side stream after that point."""
        import torch
        if self._launched[i]:
            raise RuntimeError(f"group {i} was already stepped in this step")
        producer = stream if stream is not None else torch.cuda.current_stream(self.device)
        self._ready[i].record(producer)
        self.side.wait_event(self._ready[i])
        self.step_fn(self.groups[i], self.hp, self.workspaces[i], stream=self.side)
        self._launched[i] = True

    def wait(self, stream=None) -> None:
        """`stream` (default: current) waits for every group stepped so far;
        every group must have been stepped. Starts the next step."""
        import torch
        missing = [i for i, done in enumerate(self._launched) if not done]
        if missing:
            raise RuntimeError(f"groups {missing} were not stepped")
        consumer = stream if stream is not None else torch.cuda.current_stream(self.device)
        self._done.record(self.side)
        consumer.wait_event(self._done)
        self._launched = [False] * len(self.groups)

    def device_status(self) -> int:
        """Synchronises and returns the first non-zero device status of the groups."""
        from . import device_status
        for ws in self.workspaces:
            st = device_status(ws, stream=self.side)
            if st:
                return st
        return 0

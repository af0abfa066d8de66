"""Drive a synthetic workload's schedule on a ThinKVCache (GPU).

The schedule (prefill appends in calls of <= 4096 positions per sequence, one
evict to budget, optional appends and churn steps) comes from ``workloads``;
this module only turns it into library calls.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np
import torch

from . import workloads as W
from .binding import ThinKVCache


def geometry(w: W.Workload, sched: W.Schedule) -> dict:
    """Pool and table sizes that can never run out for this schedule.

    Pages are never released, so (sequence, class) needs at most
    ceil(tokens of that class ever appended / 16) pages.
    """
    pool = [0, 0, 0]
    max_blocks = 1
    for s in range(w.batch):
        tags = sched.tags(s)
        cnt = np.bincount(tags, minlength=3)
        pages = [int(math.ceil(int(cnt[c]) / 16)) for c in range(3)]
        for c in range(3):
            pool[c] += pages[c]
        max_blocks = max(max_blocks, sum(pages))
    return {"pool_pages": [max(1, p) for p in pool], "max_blocks_per_seq": max_blocks,
            "max_seqs": w.batch}


def to_dev(a, dtype, device):
    return torch.as_tensor(np.ascontiguousarray(a)).to(device=device, dtype=dtype)


class WorkloadRun:
    """A cache plus the bookkeeping of how many tokens each sequence generated."""

    def __init__(self, w: W.Workload, extra: int = 0, device: str = "cuda",
                 bits: Optional[tuple] = None):
        self.w = w
        self.sched = W.Schedule(w, extra)
        self.geom = geometry(w, self.sched)
        self.device = torch.device(device)
        self.cache = ThinKVCache(w.num_q_heads, w.num_kv_heads, w.head_dim, w.group_size,
                                 bits or w.bits, self.geom["max_seqs"],
                                 self.geom["max_blocks_per_seq"], self.geom["pool_pages"],
                                 device=device, fmt=w.fmt)
        self.generated = self.sched.lengths.astype(np.int64).copy()
        self.all_seqs = torch.arange(w.batch, dtype=torch.int32, device=self.device)

    # -- single operations --
    def append_call(self, call: W.AppendCall):
        k, v = W.call_kv(self.w, call, device=self.device)
        self.cache.append(to_dev(call.seqs, torch.int32, self.device),
                          to_dev(call.pos, torch.int32, self.device),
                          to_dev(call.tags, torch.uint8, self.device), k, v)

    def evict_all(self):
        b = self.sched.budgets(self.generated)
        self.cache.evict(self.all_seqs, to_dev(b, torch.int32, self.device))

    def decode(self, step: int, topk: Optional[int] = None):
        q = W.q_values(self.w, step, device=self.device)
        return self.cache.decode(self.all_seqs, q, topk=topk)

    # -- schedule --
    def setup(self):
        for call in self.sched.prefill_calls():
            self.append_call(call)
        self.evict_all()
        post = self.sched.post_evict_call()
        if post is not None:
            self.append_call(post)
            self.generated += self.w.post_evict_append
        for _ in range(self.w.churn_steps):
            self.churn_step(decode=False)

    def churn_step(self, decode: bool = False, step: int = 0, topk: Optional[int] = None):
        call = self.sched.one_token_call(self.generated)
        self.append_call(call)
        self.generated += 1
        self.evict_all()
        if decode:
            return self.decode(step, topk)
        return None


# --------------------------------------------------------------------------- #
# decode steps: one token appended per sequence, evict to budget, decode
# --------------------------------------------------------------------------- #
class StepInputs:
    """Everything one step consumes, as tensors on one device (or pinned host)."""

    FIELDS = ("seqs", "pos", "tags", "k", "v", "budgets", "q")

    def __init__(self, **t):
        for f in self.FIELDS:
            setattr(self, f, t[f])

    def nbytes(self) -> int:
        return sum(getattr(self, f).numel() * getattr(self, f).element_size() for f in self.FIELDS)

    def to(self, device, pin: bool = False) -> "StepInputs":
        out = {}
        for f in self.FIELDS:
            x = getattr(self, f).to(device)
            out[f] = x.pin_memory() if pin else x
        return StepInputs(**out)


class PackedStep:
    """A step's inputs as views into one contiguous byte buffer (host, pinned
    host or device), so that moving a step between host and device is a
    single copy.  Every field starts on a 256-byte boundary."""

    ALIGN = 256

    def __init__(self, like: StepInputs, device, pin: bool = False):
        layout, off = [], 0
        for f in StepInputs.FIELDS:
            t = getattr(like, f)
            n = t.numel() * t.element_size()
            layout.append((f, off, n, t.dtype, tuple(t.shape)))
            off += (n + self.ALIGN - 1) // self.ALIGN * self.ALIGN
        buf = torch.empty(max(off, self.ALIGN), dtype=torch.uint8, device=device)
        self.buf = buf.pin_memory() if pin else buf
        self.inputs = StepInputs(**{f: self.buf[o:o + n].view(dt).view(shape)
                                    for f, o, n, dt, shape in layout})

    def fill(self, src: StepInputs) -> "PackedStep":
        """Copies ``src`` in, field by field (synchronous; for setup only)."""
        for f in StepInputs.FIELDS:
            getattr(self.inputs, f).copy_(getattr(src, f))
        return self

    def nbytes(self) -> int:
        return self.buf.numel()


def make_steps(run: "WorkloadRun", nsteps: int, first_step: int = 0, device=None):
    """Inputs of the next ``nsteps`` steps of ``run`` (does not advance it)."""
    w = run.w
    device = run.device if device is None else device
    gen = run.generated.copy()
    steps = []
    for k in range(nsteps):
        call = run.sched.one_token_call(gen)
        kk, vv = W.call_kv(w, call, device=device)
        gen = gen + 1
        steps.append(StepInputs(
            seqs=to_dev(call.seqs, torch.int32, device), pos=to_dev(call.pos, torch.int32, device),
            tags=to_dev(call.tags, torch.uint8, device), k=kk, v=vv,
            budgets=to_dev(run.sched.budgets(gen), torch.int32, device),
            q=W.q_values(w, first_step + k, device=device)))
    return steps


def run_step(cache: ThinKVCache, inp: StepInputs, out: torch.Tensor, topk: Optional[int] = None,
             mass: Optional[torch.Tensor] = None):
    """One step on device-resident inputs: append + evict to budget (one call:
    one token per sequence, the budgets in the same order), then decode."""
    cache.append_evict(inp.seqs, inp.pos, inp.tags, inp.k, inp.v, inp.budgets)
    return cache.decode(inp.seqs, inp.q, topk=topk, out=out, mass=mass)


def run_step_from_host(cache: ThinKVCache, host: PackedStep, dev: PackedStep,
                       out_dev: torch.Tensor, out_host: torch.Tensor, topk: Optional[int] = None,
                       mass_dev: Optional[torch.Tensor] = None,
                       mass_host: Optional[torch.Tensor] = None):
    """One step whose inputs start in pinned host memory and whose outputs end
    there: one host->device copy of the packed inputs, the two library
    calls, device->host copies, all queued on the current stream."""
    dev.buf.copy_(host.buf, non_blocking=True)
    run_step(cache, dev.inputs, out_dev, topk=topk, mass=mass_dev)
    out_host.copy_(out_dev, non_blocking=True)
    if topk:
        mass_host.copy_(mass_dev, non_blocking=True)

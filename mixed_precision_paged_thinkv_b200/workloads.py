"""Seeded synthetic workloads for the ThinKV decode hot path.

This module only *generates inputs*: sequence lengths, thought-type tags
(R=0, E=1, T=2), K/V/Q values and the call schedule.  It holds none of the
method's arithmetic (no quantisation, no eviction, no attention), so both the
CPU oracle (``oracle/``) and the CUDA library can be fed from it.

The workloads are synthetic stand-ins for the long chain-of-thought decodes the
ThinKV pages evaluate on (DeepSeek-R1-Distill, GPT-OSS, AceReason on AIME /
LiveCodeBench / MATH-500; "ThinKV: Thought-Adaptive KV Cache Compression for
Efficient Reasoning Models", arXiv abstract and the explainer's "Résumé
Technique / Résultats").  Shapes, lengths and the tag process follow the five
named layer configurations; see ``WORKLOADS``.

Values.  K, V and Q are fp16 with an approximately standard-normal
distribution: each value is the textbook "sum of twelve uniforms minus six"
(Irwin-Hall(12)), built from a counter-based 32-bit integer hash so that the
same values come out bit-for-bit on CPU and on GPU tensors (every step is an
integer op, an exact int->fp32 conversion, an exact power-of-two scale and one
fp32->fp16 round-to-nearest).  Outlier (kv-head, channel) pairs are multiplied
by 8 before the fp16 rounding.  Q has no outliers.

Tags.  Each sequence's positions are cut into segments; segment lengths are
uniform on {16..64} for the tiny case and Geometric(p=1/40) on {1,2,...}
otherwise; each segment's tag is drawn i.i.d. with probabilities
R/E/T = 0.3/0.5/0.2.  These small arrays come from ``numpy.random.default_rng``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

TAG_R, TAG_E, TAG_T = 0, 1, 2
PAGE_SIZE = 16

_M32 = 0xFFFFFFFF


# --------------------------------------------------------------------------- #
# workload descriptions
# --------------------------------------------------------------------------- #
@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload (a single attention layer)."""

    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    group_size: int
    bits: Tuple[int, int, int] = (8, 4, 2)
    # code format per class: 0 integer asymmetric codes, 1 the float formats
    # (FP8 E4M3 / FP4 E2M1 / ternary at 8 / 4 / 2 bits)
    fmt: Tuple[int, int, int] = (0, 0, 0)
    page_size: int = PAGE_SIZE
    # sequence lengths: ("fixed", n) | ("uniform", lo, hi) | ("loguniform", lo, hi)
    lengths: tuple = ("fixed", 512)
    # segment process: ("uniform", lo, hi) | ("geometric", mean)
    segments: tuple = ("geometric", 40)
    tag_probs: Tuple[float, float, float] = (0.3, 0.5, 0.2)
    # budget: ("fixed", n) | ("frac", f)
    budget: tuple = ("frac", 0.05)
    # outliers: ("count", n) | ("frac", f)  -- (kv-head, channel) pairs x8
    outliers: tuple = ("frac", 0.01)
    # tokens appended (one call, all sequences) right after the setup evict
    post_evict_append: int = 0
    # (append 1 token / sequence, evict) steps run after setup
    churn_steps: int = 0
    # the fused top-k attention-mass statistic is requested
    topk: Optional[int] = None
    # oracle check cadence during churn (0 = only at the end)
    check_every: int = 0
    seed: int = 0
    # largest number of positions of one sequence in one setup append call
    setup_call_positions: int = 4096

    @property
    def gq(self) -> int:
        return self.num_q_heads // self.num_kv_heads


WORKLOADS = {
    "tiny": Workload(
        name="tiny", batch=1, num_q_heads=4, num_kv_heads=2, head_dim=64,
        group_size=32, lengths=("fixed", 512), segments=("uniform", 16, 64),
        budget=("fixed", 256), outliers=("count", 4), post_evict_append=64,
        seed=0),
    "r1-llama-8b": Workload(
        name="r1-llama-8b", batch=16, num_q_heads=32, num_kv_heads=8,
        head_dim=128, group_size=64, lengths=("fixed", 16384),
        segments=("geometric", 40), budget=("frac", 0.05), seed=1),
    "r1-qwen-14b": Workload(
        name="r1-qwen-14b", batch=32, num_q_heads=40, num_kv_heads=8,
        head_dim=128, group_size=64, lengths=("fixed", 32768),
        segments=("geometric", 40), budget=("frac", 0.05), churn_steps=128,
        seed=2),
    "gpt-oss-20b": Workload(
        name="gpt-oss-20b", batch=64, num_q_heads=64, num_kv_heads=8,
        head_dim=64, group_size=32, lengths=("uniform", 8192, 32768),
        segments=("geometric", 40), budget=("frac", 0.10), topk=32, seed=3),
    "churn": Workload(
        name="churn", batch=128, num_q_heads=32, num_kv_heads=8,
        head_dim=128, group_size=64, lengths=("loguniform", 2048, 65536),
        segments=("geometric", 40), budget=("frac", 0.05), churn_steps=1000,
        check_every=100, seed=4),
}
WORKLOAD_ORDER = ["tiny", "r1-llama-8b", "r1-qwen-14b", "gpt-oss-20b", "churn"]


def before_eviction(w: Workload) -> Workload:
    """The same layer shape and history, timed before any eviction: every
    generated token stays live, with the segment tag mix (R/E/T about
    0.3/0.5/0.2), so the 4-bit and 2-bit pages are read at full scale.  The
    retained state of the budgeted workloads is almost all R (8-bit)."""
    return dataclasses.replace(w, name=w.name + "-mixed", budget=("frac", 1.0), churn_steps=0,
                               check_every=0)


def float_formats(w: Workload) -> Workload:
    """The same layer and history with the pages' own code formats: FP8 E4M3
    for R, FP4 E2M1 for E, ternary for T (the explainer's TBQ)."""
    return dataclasses.replace(w, name=w.name + "-float", fmt=(1, 1, 1))


# Supplementary measurements (not the headline configurations).
SUPPLEMENTARY = {n + "-mixed": before_eviction(WORKLOADS[n])
                 for n in ("r1-llama-8b", "r1-qwen-14b", "gpt-oss-20b", "churn")}
SUPPLEMENTARY.update({n + "-float": float_formats(WORKLOADS[n])
                      for n in ("r1-llama-8b", "churn")})
SUPPLEMENTARY["r1-llama-8b-mixed-float"] = float_formats(before_eviction(WORKLOADS["r1-llama-8b"]))


def get(name: str) -> Workload:
    """A workload by name: the five configurations, or a supplementary one."""
    if name in WORKLOADS:
        return WORKLOADS[name]
    if name in SUPPLEMENTARY:
        return SUPPLEMENTARY[name]
    raise KeyError(f"unknown workload {name!r}")


def scaled(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (used for reduced test cases)."""
    return dataclasses.replace(w, **kw)


# --------------------------------------------------------------------------- #
# small host-side arrays (numpy)
# --------------------------------------------------------------------------- #
def _rng(w: Workload, *stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([w.seed, *stream]))


def seq_lengths(w: Workload) -> np.ndarray:
    """History length (tokens generated before the first decode) per sequence."""
    kind = w.lengths[0]
    if kind == "fixed":
        return np.full(w.batch, int(w.lengths[1]), dtype=np.int64)
    rng = _rng(w, 1)
    if kind == "uniform":
        lo, hi = int(w.lengths[1]), int(w.lengths[2])
        return rng.integers(lo, hi + 1, size=w.batch).astype(np.int64)
    if kind == "loguniform":
        lo, hi = float(w.lengths[1]), float(w.lengths[2])
        u = rng.uniform(math.log(lo), math.log(hi), size=w.batch)
        return np.floor(np.exp(u)).astype(np.int64)
    raise ValueError(kind)


def seq_tags(w: Workload, seq: int, n: int) -> np.ndarray:
    """Thought-type tags of positions 0..n-1 of sequence ``seq`` (uint8)."""
    rng = _rng(w, 2, seq)
    out = np.empty(n, dtype=np.uint8)
    filled = 0
    probs = np.asarray(w.tag_probs, dtype=np.float64)
    while filled < n:
        if w.segments[0] == "uniform":
            ln = int(rng.integers(int(w.segments[1]), int(w.segments[2]) + 1))
        else:
            ln = int(rng.geometric(1.0 / float(w.segments[1])))
        tag = int(rng.choice(3, p=probs))
        end = min(n, filled + ln)
        out[filled:end] = tag
        filled = end
    return out


def outlier_pairs(w: Workload) -> np.ndarray:
    """(kv_head, channel) pairs whose K and V values are scaled by 8."""
    hd = w.num_kv_heads * w.head_dim
    if w.outliers[0] == "count":
        n = int(w.outliers[1])
    else:
        n = max(1, int(round(float(w.outliers[1]) * hd)))
    rng = _rng(w, 3)
    flat = rng.choice(hd, size=n, replace=False)
    return np.stack([flat // w.head_dim, flat % w.head_dim], axis=1).astype(np.int64)


def budget_for(w: Workload, generated: int) -> int:
    """Token budget of a sequence that has generated ``generated`` tokens."""
    if w.budget[0] == "fixed":
        return int(w.budget[1])
    return max(1, int(math.floor(float(w.budget[1]) * generated)))


# --------------------------------------------------------------------------- #
# counter-based values (torch integer ops; identical on CPU and GPU)
# --------------------------------------------------------------------------- #
def _mul32(a: torch.Tensor, c: int) -> torch.Tensor:
    """(a * c) mod 2**32 for 0 <= a < 2**32, without int64 overflow."""
    lo = a * (c & 0xFFFF)
    hi = (a * (c >> 16)) & 0xFFFF
    return (lo + (hi << 16)) & _M32


def _mix32(x: torch.Tensor) -> torch.Tensor:
    """A 32-bit integer finaliser (xorshift-multiply, 'lowbias32' constants)."""
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


_STREAM_KV, _STREAM_Q = 11, 12


def _normal_fp16_from_ids(ids: torch.Tensor, seed: int, stream: int) -> torch.Tensor:
    """Approximately N(0,1) fp16 values, one per int64 counter in ``ids``."""
    salt = (seed * 0x9E3779B1 + stream * 0x85EBCA77 + 0x165667B1) & _M32
    lo = ids & _M32
    hi = (ids >> 32) & _M32
    base = _mix32(lo ^ _mix32(hi ^ salt))
    acc = torch.zeros_like(ids)
    for j in range(6):
        r = _mix32(base ^ ((0x27D4EB2F * (j + 1) + salt) & _M32))
        acc = acc + (r & 0xFFFF) + (r >> 16)
    # twelve 16-bit uniforms: mean 12*32767.5, sd ~= 65536
    centred = (acc - 393210).to(torch.float32)
    return (centred * (1.0 / 65536.0)).to(torch.float16)


def kv_for_tokens(w: Workload, seqs, pos, device="cpu",
                  chunk_tokens: int = 1 << 14) -> Tuple[torch.Tensor, torch.Tensor]:
    """K and V (fp16, shape [n, Hkv, d]) of the tokens (seqs[i], pos[i]).

    Every value is a function of (seed, sequence, position, head, channel, K|V)
    only, so any subset of tokens can be regenerated on any device."""
    H, d = w.num_kv_heads, w.head_dim
    per_tok = H * d * 2
    seqs_t = torch.as_tensor(np.asarray(seqs, dtype=np.int64), device=device)
    pos_t = torch.as_tensor(np.asarray(pos, dtype=np.int64), device=device)
    n = int(seqs_t.numel())
    out = torch.empty(n, per_tok, dtype=torch.float16, device=device)
    lane = torch.arange(per_tok, dtype=torch.int64, device=device)
    for a in range(0, n, chunk_tokens):
        b = min(n, a + chunk_tokens)
        base = ((seqs_t[a:b] << 26) + pos_t[a:b]) * per_tok
        ids = base[:, None] + lane[None, :]
        out[a:b] = _normal_fp16_from_ids(ids, w.seed, _STREAM_KV)
    kv = out.view(n, H, d, 2)
    pairs = outlier_pairs(w)
    if len(pairs) and n:
        hh = torch.as_tensor(pairs[:, 0], device=device)
        cc = torch.as_tensor(pairs[:, 1], device=device)
        kv32 = kv[:, hh, cc, :].to(torch.float32) * 8.0
        kv[:, hh, cc, :] = kv32.to(torch.float16)
    return kv[..., 0].contiguous(), kv[..., 1].contiguous()


def kv_values(w: Workload, seq: int, pos0: int, n: int,
              device="cpu") -> Tuple[torch.Tensor, torch.Tensor]:
    """K and V (fp16, shape [n, Hkv, d]) of positions pos0..pos0+n-1 of ``seq``."""
    return kv_for_tokens(w, np.full(n, seq, dtype=np.int64), np.arange(pos0, pos0 + n), device)


def q_values(w: Workload, step: int, device="cpu") -> torch.Tensor:
    """Decode queries (fp16, [batch, Hq, d]) of decode step ``step``."""
    B, Hq, d = w.batch, w.num_q_heads, w.head_dim
    n = B * Hq * d
    ids = torch.arange(n, dtype=torch.int64, device=device) + step * n
    return _normal_fp16_from_ids(ids, w.seed, _STREAM_Q).view(B, Hq, d)


# --------------------------------------------------------------------------- #
# call schedule
# --------------------------------------------------------------------------- #
@dataclasses.dataclass
class AppendCall:
    """One append call: tokens grouped by sequence, positions ascending."""

    seqs: np.ndarray   # int32 [n] sequence id per token
    pos: np.ndarray    # int32 [n] position per token
    tags: np.ndarray   # uint8 [n]
    runs: List[Tuple[int, int, int]]  # (seq, pos0, count) in call order

    @property
    def n(self) -> int:
        return int(self.seqs.shape[0])


def make_append_call(runs: Sequence[Tuple[int, int, int]], tags_of) -> AppendCall:
    """Build an append call from (seq, pos0, count) runs; ``tags_of(seq)`` gives tags."""
    seqs, pos, tags = [], [], []
    for (s, p0, c) in runs:
        seqs.append(np.full(c, s, dtype=np.int32))
        pos.append(np.arange(p0, p0 + c, dtype=np.int32))
        tags.append(tags_of(s)[p0:p0 + c])
    if not runs:
        z = np.zeros(0, dtype=np.int32)
        return AppendCall(z, z.copy(), np.zeros(0, dtype=np.uint8), [])
    return AppendCall(np.concatenate(seqs), np.concatenate(pos),
                      np.concatenate(tags).astype(np.uint8), list(runs))


def call_kv(w: Workload, call: AppendCall, device="cpu") -> Tuple[torch.Tensor, torch.Tensor]:
    """K and V ([n, Hkv, d] fp16) of every token of ``call``, in call order."""
    return kv_for_tokens(w, call.seqs, call.pos, device=device)


class Schedule:
    """The setup of a workload: prefill appends, one evict, optional appends.

    ``extra`` positions per sequence are reserved beyond the history for the
    tokens appended after setup (post-evict appends, churn steps, timed steps),
    so that tags exist for them.
    """

    def __init__(self, w: Workload, extra: int = 0):
        self.w = w
        self.lengths = seq_lengths(w)
        self.extra = int(extra) + w.post_evict_append + w.churn_steps
        self._tags = {}

    def tags(self, seq: int) -> np.ndarray:
        t = self._tags.get(seq)
        if t is None:
            t = seq_tags(self.w, seq, int(self.lengths[seq]) + self.extra)
            self._tags[seq] = t
        return t

    def prefill_calls(self) -> List[AppendCall]:
        w = self.w
        step = w.setup_call_positions
        longest = int(self.lengths.max()) if len(self.lengths) else 0
        calls = []
        for p0 in range(0, longest, step):
            runs = []
            for s in range(w.batch):
                L = int(self.lengths[s])
                if p0 < L:
                    runs.append((s, p0, min(step, L - p0)))
            calls.append(make_append_call(runs, self.tags))
        return calls

    def budgets(self, generated: np.ndarray) -> np.ndarray:
        return np.asarray([budget_for(self.w, int(g)) for g in generated], dtype=np.int32)

    def one_token_call(self, generated: np.ndarray) -> AppendCall:
        """One new token per sequence, at position ``generated[s]``."""
        runs = [(s, int(generated[s]), 1) for s in range(self.w.batch)]
        return make_append_call(runs, self.tags)

    def post_evict_call(self) -> Optional[AppendCall]:
        w = self.w
        if w.post_evict_append <= 0:
            return None
        runs = [(s, int(self.lengths[s]), w.post_evict_append) for s in range(w.batch)]
        return make_append_call(runs, self.tags)


def algorithmic_decode_bytes(w: Workload, live_by_class: Sequence[int],
                             table_entries: int, with_stat: bool) -> int:
    """Bytes a decode call must move at minimum (live tokens, table, Q, O, stat).

    ``live_by_class[c]`` is the number of live tokens of class c over all
    decoded sequences; each is counted once per kv-head.
    """
    d, G, H = w.head_dim, w.group_size, w.num_kv_heads
    total = 0
    for c, n in enumerate(live_by_class):
        b = w.bits[c]
        per = 2 * d * b // 8
        if b < 16:
            per += 2 * (d // G) * 4
        total += int(n) * H * per
    total += int(table_entries) * 8
    total += 2 * w.batch * w.num_q_heads * d * 2
    if with_stat:
        total += w.batch * w.num_q_heads * 4
    return total

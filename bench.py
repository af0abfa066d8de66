"""Benchmark of the ThinKV decode hot path (append -> evict -> decode per step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl thinkv|reference]

One step = one token appended (quantised) per sequence, eviction back to the
budget, and decode attention (+ the top-k mass when the workload asks for
it) over every sequence -- the whole hot path over one batch.  The workload
defaults to the serving-churn layer, the largest single-GPU configuration
(128 sequences with lengths log-uniform over 2k-64k, 1000 churn steps before
timing, 32/8 heads, head_dim 128, 8/4/2-bit R/E/T codes, group 64, 5%
budget).  In the same run the three other budgeted layer shapes
(R1-Distill-Llama-8B, R1-Distill-Qwen-14B, GPT-OSS-20B) are set up and timed
the same way; their lines go to `per_config`.  Inputs are synthetic and
seeded; the per-step inputs are resident on the GPU before timing; L2 is
flushed (512 MiB write) between steps, outside the timed events.

The metric is decode tokens/s (one token per sequence per step); the
roofline block reports the decode kernel's achieved HBM bandwidth from its
algorithmic bytes.  `--impl reference` times the CPU oracle (oracle/) on the
same workload.  Multi-GPU: replicas only (each rank runs its own copy of the
workload; no data-path collective); value = tokens of all ranks / max time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-attention tokens/sec and achieved HBM GB/s (% of B200 peak), 1 GPU"
DEFAULT_WORKLOAD = "churn"
PER_CONFIG = ["r1-llama-8b", "r1-qwen-14b", "gpt-oss-20b"]
FLUSH_BYTES = 512 << 20
# the sources the decode kernels are compiled from (the shared internal header
# holds host-side declarations only)
DECODE_SRC = [os.path.join(ROOT, "mixed_precision_paged_thinkv_b200", "csrc", f)
              for f in ("thinkv_decode.cu", "thinkv_common.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1000 * 1000    # B200 L2: a step reading more than this cannot run from L2


# --------------------------------------------------------------------------- #
# small host-side helpers (unit-tested on CPU)
# --------------------------------------------------------------------------- #
def aggregate(per_rank):
    """per_rank: [(tokens, seconds)] -> (total tokens / max seconds, max seconds)."""
    tokens = sum(t for t, _ in per_rank)
    worst = max(s for _, s in per_rank)
    return tokens / worst, worst


def parse_clocks(csv_text: str, index: int = None):
    """Summary of `nvidia-smi --query-gpu=index,clocks.sm,clocks.max.sm,power.draw,
    clocks_event_reasons.active,...hw_slowdown,hw_thermal_slowdown,sw_thermal_slowdown,
    sw_power_cap --format=csv` samples taken during the timed region."""
    rows = []
    for line in csv_text.strip().splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9 or not parts[0].isdigit():
            continue
        if index is not None and int(parts[0]) != index:
            continue
        try:
            sm = float(parts[1].split()[0])
            smax = float(parts[2].split()[0])
        except ValueError:
            continue
        rows.append((sm, smax, parts[5:9]))
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[k] for (_, _, flags) in rows for k, f in enumerate(flags)
                      if f.lower().startswith("active")})
    sm = sorted(r[0] for r in rows)
    return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[1] for r in rows),
            "reasons": reasons, "samples": len(rows)}


def peak_hbm_gbs():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def decode_source_hash() -> str:
    """Hash of the sources the decode kernel is compiled from."""
    h = hashlib.sha256()
    for p in DECODE_SRC:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_per_launch(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current decode source for this workload; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        e = rec.get(workload)
        if e and e.get("source_sha") == decode_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def launches_per_step(batch: int) -> int:
    """Kernels one step launches: append + evict (one launch up to 512 tokens,
    else the append's two and the evict's one), decode (split + combine)."""
    return (1 if batch <= 512 else 3) + 2


def algorithmic_decode_bytes(w, snap) -> int:
    """Bytes one decode call must move: codes + params of every live token for
    every kv-head, the table entry and live-list entry (8 B each) of every
    live page, the sequence id and live-page count (4 B each) of every
    sequence, Q, O and (if asked) the fp32 top-k mass."""
    H, d, G = w.num_kv_heads, w.head_dim, w.group_size

    def entry_class(e):  # block-table entry: page | class << 32 | live_mask << 48
        return (int(e) >> 32) & 0xFF

    def entry_mask(e):
        return (int(e) >> 48) & 0xFFFF

    live_by_class = [0, 0, 0]
    pages = 0
    for s in range(w.batch):
        nl = int(snap["num_live"][s])
        desc = snap["live_list"][s, :nl]            # page | class << 32 | entry << 40
        ents = snap["table"][s, (desc >> np.uint64(40)).astype(np.int64)]
        pages += nl
        for e in ents:
            live_by_class[int(entry_class(e))] += bin(int(entry_mask(e))).count("1")
    total = 0
    for c in range(3):
        b = w.bits[c]
        per = 2 * d * b // 8 + (2 * (d // G) * 4 if b < 16 else 0)
        total += live_by_class[c] * H * per
    total += pages * (8 + 8)
    total += w.batch * (4 + 4)
    total += 2 * w.batch * w.num_q_heads * d * 2
    if w.topk:
        total += w.batch * w.num_q_heads * 4
    return total, live_by_class, pages


class ClockSampler:
    QUERY = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, out_path):
        self.out_path = out_path
        self.proc = None

    def start(self):
        try:
            self.f = open(self.out_path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}",
                                          "--format=csv", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, uuid: str):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        text = open(self.out_path).read()
        # drop the uuid column after selecting our GPU's rows
        keep = []
        for line in text.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 10 and parts[0].isdigit():
                u = parts[1].replace("GPU-", "")
                if uuid and u != uuid.replace("GPU-", ""):
                    continue
                keep.append(",".join([parts[0]] + parts[2:]))
        return parse_clocks("\n".join(keep))


# --------------------------------------------------------------------------- #
# distributed plumbing (replicas only)
# --------------------------------------------------------------------------- #
def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if os.environ.get("THINKV_BENCH_BACKEND", "nccl") == "nccl" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def dist_max_sum(seconds: float, tokens: float, world: int, device):
    if world == 1:
        return seconds, tokens
    import torch
    import torch.distributed as dist
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    n = torch.tensor([tokens], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), float(n.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------------- #
# oracle timing (CPU baseline and the reference arm)
# --------------------------------------------------------------------------- #
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def sample_sequences(w, n_sample: int):
    """An evenly spaced sample of the workload's sequences (all if it has fewer):
    the CPU legs replay only these, so their cost stays bounded."""
    if w.batch <= n_sample:
        return list(range(w.batch))
    return [int(x) for x in np.linspace(0, w.batch - 1, n_sample).round().astype(int)]


class OracleReplay:
    """The oracle replaying a sample of a workload's sequences: the same
    prefill calls, setup evict, churn steps and timed steps as the GPU run,
    restricted to those sequences.  Sequences never interact (except through
    the numbering of pages), so each step's work per sequence is the work of
    the full-batch run; throughput scales by sequences."""

    def __init__(self, w, seqs, extra: int, gen_device: str):
        import math as _m
        from mixed_precision_paged_thinkv_b200 import workloads as W
        from oracle import oracle as O
        self.W, self.O = W, O
        self.w, self.seqs, self.gen_device = w, list(seqs), gen_device
        self.sched = W.Schedule(w, extra)
        pool, mb = [0, 0, 0], 1
        for s in self.seqs:
            cnt = np.bincount(self.sched.tags(s), minlength=3)
            pages = [int(_m.ceil(int(cnt[c]) / 16)) for c in range(3)]
            pool = [a + b for a, b in zip(pool, pages)]
            mb = max(mb, sum(pages))
        self.o = O.Oracle(w.num_q_heads, w.num_kv_heads, w.head_dim, w.group_size, w.bits,
                          len(self.seqs), mb, [max(1, p) for p in pool], fmt=w.fmt)
        self.generated = self.sched.lengths[self.seqs].astype(np.int64).copy()
        self.ids = np.arange(len(self.seqs), dtype=np.int32)

    def _append(self, runs):
        W, O = self.W, self.O
        if not runs:
            return
        S, P, T, orig = [], [], [], []
        for (j, p0, c) in runs:
            s = self.seqs[j]
            S.append(np.full(c, j, dtype=np.int32))
            P.append(np.arange(p0, p0 + c, dtype=np.int32))
            T.append(self.sched.tags(s)[p0:p0 + c])
            orig.append(np.full(c, s, dtype=np.int64))
        S, P, T, orig = map(np.concatenate, (S, P, T, orig))
        k, v = W.kv_for_tokens(self.w, orig, P.astype(np.int64), device=self.gen_device)
        assert self.o.append(S, P, T.astype(np.uint8), k.cpu(), v.cpu()) == O.OK

    def setup(self):
        where = {s: j for j, s in enumerate(self.seqs)}
        for call in self.sched.prefill_calls():
            self._append([(where[s], p0, c) for (s, p0, c) in call.runs if s in where])
        assert self.o.evict(self.ids, self.sched.budgets(self.generated)) == self.O.OK
        if self.w.post_evict_append:
            n = self.w.post_evict_append
            self._append([(j, int(self.generated[j]), n) for j in range(len(self.seqs))])
            self.generated += n
        for _ in range(self.w.churn_steps):
            self.step_inputs_and_run(0, decode=False)

    def step_inputs(self, step: int):
        """The next step's inputs: one token per sampled sequence, budgets, Q rows."""
        W = self.W
        pos = self.generated.astype(np.int32)
        tags = np.array([self.sched.tags(s)[int(p)] for s, p in zip(self.seqs, pos)], np.uint8)
        k, v = W.kv_for_tokens(self.w, np.asarray(self.seqs, np.int64), pos.astype(np.int64),
                               device=self.gen_device)
        budgets = self.sched.budgets(self.generated + 1)
        q = W.q_values(self.w, step, device=self.gen_device)[self.seqs].cpu()
        return pos, tags, k.cpu(), v.cpu(), budgets, q

    def run_step(self, inp, threads: int, decode: bool = True):
        """append + evict (+ decode); returns (step seconds, decode seconds)."""
        O = self.O
        pos, tags, k, v, budgets, q = inp
        t0 = time.perf_counter()
        assert self.o.append(self.ids, pos, tags, k, v) == O.OK
        assert self.o.evict(self.ids, budgets) == O.OK
        t1 = time.perf_counter()
        if decode:
            self.o.decode(self.ids, q, topk=self.w.topk, threads=threads)
        t2 = time.perf_counter()
        self.generated += 1
        return t2 - t0, t2 - t1

    def step_inputs_and_run(self, step, decode=True, threads=1):
        return self.run_step(self.step_inputs(step), threads, decode)


def time_oracle(w, steps: int, warmup: int, budget_s: float, gen_device: str,
                n_sample: int = 0, repeats: int = 5):
    """The oracle as it stands, on a bounded sample of the workload: the
    sampled sequences' setup is replayed untimed, then steps (append 1 token
    per sequence + evict + decode) are timed.  Each step is timed with the
    decode on all host cores and, on a copy of the same inputs, the decode
    alone single-threaded is timed too.  Medians over up to `repeats` steps
    (at least one), stopping once `budget_s` of timed work is spent."""
    # one sampled sequence per host core at least: decode parallelises over sequences
    seqs = sample_sequences(w, n_sample or max(8, os.cpu_count() or 1))
    rep = OracleReplay(w, seqs, extra=warmup + steps + repeats + 4, gen_device=gen_device)
    t0 = time.time()
    rep.setup()
    setup_s = time.time() - t0
    threads = os.cpu_count() or 1
    for k in range(warmup):
        rep.step_inputs_and_run(k, threads=threads)
    step_s, dec_s, dec1_s = [], [], []
    spent = 0.0
    for k in range(max(1, min(steps, repeats))):
        inp = rep.step_inputs(warmup + k)
        st, dt = rep.run_step(inp, threads)
        # the same decode again, single-threaded (the state did not change)
        t = time.perf_counter()
        rep.o.decode(rep.ids, inp[5], topk=w.topk, threads=1)
        d1 = time.perf_counter() - t
        step_s.append(st)
        dec_s.append(dt)
        dec1_s.append(d1)
        spent += st + d1
        if spent > budget_s:
            break
    med = lambda x: float(np.median(x))
    n = len(seqs)
    return {"value": n / med(step_s), "decode_tokens_per_s": n / med(dec_s),
            "decode_tokens_per_s_1thread": n / med(dec1_s),
            "step_ms": 1000 * med(step_s), "steps": len(step_s), "cores": threads,
            "seqs": n, "setup_s": setup_s, "seconds": float(sum(step_s))}


def _oracle_sample_text(w, r) -> str:
    return (f"oracle (C, fp64 attention) on {r['seqs']} of {w.batch} sequences (evenly spaced), "
            f"their setup replayed untimed; median of {r['steps']} steps of append 1 token/seq + "
            f"evict + decode (decode on {r['cores']} OpenMP threads); tokens/s scaled per sequence; "
            f"host CPU: {cpu_model()}")


def reference_arm(args, w, world, rank):
    if rank != 0:
        return 0
    gen_device = "cuda" if _cuda_ok() else "cpu"
    r = time_oracle(w, max(args.steps, 1), min(args.warmup, 3), budget_s=60.0,
                    gen_device=gen_device)
    line = {
        "impl": "reference", "metric": METRIC, "value": r["value"], "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": r["steps"], "warmup": args.warmup,
        "ms_per_step": r["step_ms"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "dtype_detail": "attention in f64; the quantiser in the f32 operations it is defined with",
        "data": "synthetic", "config": workload_config(w, None),
        "cpu_baseline": {"value": r["value"], "unit": "tokens/s", "cores": r["cores"],
                         "kind": "oracle", "sample": _oracle_sample_text(w, r),
                         "cpu_model": cpu_model(),
                         "decode_tokens_per_s": r["decode_tokens_per_s"],
                         "decode_tokens_per_s_1thread": r["decode_tokens_per_s_1thread"]},
        "e2e": {"value": r["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _cuda_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


L2_FLUSHED = "flushed between steps (512 MiB write, outside the timed events)"
L2_LARGER = ("not flushed: the K steps run back to back, timed as one region; each step's "
             "decode reads more than L2 holds")


def workload_config(w, live, l2: str = L2_FLUSHED):
    cfg = {"workload": f"{w.name}: layer {w.num_q_heads}q/{w.num_kv_heads}kv heads, "
                       f"head_dim {w.head_dim}, batch {w.batch}, lengths {w.lengths}, "
                       f"R/E/T {w.bits[0]}/{w.bits[1]}/{w.bits[2]}-bit"
                       + (" (FP8 E4M3 / FP4 E2M1 / ternary)" if any(w.fmt) else "")
                       + f", group {w.group_size}, "
                       f"budget {w.budget}"
                       + (f", {w.churn_steps} churn steps before timing" if w.churn_steps else "")
                       + (f", top-{w.topk} mass" if w.topk else ""),
           "batch": w.batch, "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads,
           "head_dim": w.head_dim, "group_size": w.group_size, "page_size": w.page_size,
           "bits_RET": list(w.bits), "fmt_RET": list(w.fmt), "topk": w.topk,
           "l2": l2,
           "parallelism": "replicas"}
    if live is not None:
        cfg["live_tokens_by_class"] = live
    if w.budget == ("frac", 1.0):
        cfg["state"] = "supplementary: before eviction (whole history live, mixed R/E/T)"
    return cfg


# --------------------------------------------------------------------------- #
# the library arm
# --------------------------------------------------------------------------- #
def compaction_bytes(w, live_by_class) -> int:
    """Bytes a gather compaction must move at least: every live token's codes
    and params for every kv-head, read once and written once."""
    H, d, G = w.num_kv_heads, w.head_dim, w.group_size
    per = [2 * d * b // 8 + (2 * (d // G) * 4 if b < 16 else 0) for b in w.bits]
    return 2 * sum(n * H * p for n, p in zip(live_by_class, per))


def measure_compaction(w, run, last, out, mass, live, K: int, flush, dev):
    """The step Continuous Thinking avoids: the state the timed steps left is
    gathered into fresh hole-free pages of a second cache (thinkv_compact),
    K times (the copy reset outside the events, L2 flushed), and the same
    decode call is timed on the compacted copy."""
    import torch
    from mixed_precision_paged_thinkv_b200.binding import ThinKVCache
    c = run.cache
    # sized from the state as it is now (the timed steps may have grown it)
    _, live, _ = algorithmic_decode_bytes(w, c.snapshot())
    pool = [n // 16 + w.batch + 1 for n in live]
    dst = ThinKVCache(w.num_q_heads, w.num_kv_heads, w.head_dim, w.group_size, w.bits,
                      c.max_seqs, c.max_blocks, pool, device=str(dev), fmt=w.fmt)
    max_tok = int(sum(live)) + 16 * w.batch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    for k in range(K):
        dst.reset()
        flush.zero_()
        ev[k][0].record()
        c.compact_into(dst, last.seqs, max_tok)
        ev[k][1].record()
    torch.cuda.synchronize()
    assert dst.status() == 0, "device status after compaction"
    comp_ms = [a.elapsed_time(b) for a, b in ev]
    dev_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
    for k in range(K):
        flush.zero_()
        dev_ev[k][0].record()
        dst.decode(last.seqs, last.q, topk=w.topk, out=out, mass=mass)
        dev_ev[k][1].record()
    torch.cuda.synchronize()
    dec_ms = [a.elapsed_time(b) for a, b in dev_ev]
    snap = dst.snapshot()
    _, _, pages = algorithmic_decode_bytes(w, snap)
    del dst, snap
    torch.cuda.empty_cache()
    cm = sum(comp_ms) / K
    nbytes = compaction_bytes(w, live)
    return {"kernels": "thinkv_compact (compact_count_kernel, compact_plan_kernel, compact_list_kernel, compact_copy_kernel)",
            "ms": cm, "bytes_moved_min": nbytes, "gbs": nbytes / (cm / 1000.0) / 1e9,
            "decode_ms_on_compacted": sum(dec_ms) / K, "live_pages_after": pages,
            "note": "what one step would add if it compacted after each eviction (the step "
                    "Continuous Thinking avoids), and the decode call on the compacted copy"}


def measure_workload(w, K: int, Wm: int, dev, flush, e2e_steps: int = 0, clocks=None,
                     world: int = 1, compaction: bool = False):
    """Sets the workload up on the GPU, then times K steps (append + evict +
    decode, one event pair per step, L2 flushed before each), the decode call
    alone K times on the state the steps left, and (if e2e_steps) steps from
    pinned host buffers.  Returns the measurements of this rank."""
    import torch
    from mixed_precision_paged_thinkv_b200.runner import (PackedStep, WorkloadRun, make_steps,
                                                          run_step, run_step_from_host)
    run = WorkloadRun(w, extra=Wm + K + e2e_steps + 2, device=str(dev))
    run.setup()
    torch.cuda.synchronize()
    steps = make_steps(run, Wm + K + e2e_steps, device=dev)
    out = torch.empty(w.batch, w.num_q_heads, w.head_dim, dtype=torch.float16, device=dev)
    mass = torch.empty(w.batch, w.num_q_heads, dtype=torch.float32, device=dev) if w.topk else None
    for k in range(Wm):
        flush.zero_()
        run_step(run.cache, steps[k], out, topk=w.topk, mass=mass)
    torch.cuda.synchronize()
    assert run.cache.status() == 0, "device status after warm-up"
    snap = run.cache.snapshot()
    alg_bytes, live, pages = algorithmic_decode_bytes(w, snap)
    del snap

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
        time.sleep(0.4)
    # a step that reads more than L2 holds cannot be helped by the previous
    # one's cache lines: such steps run back to back, as a serving loop does,
    # and the K steps are timed as one region; smaller ones are timed one at a
    # time with L2 flushed between them (outside the events)
    back_to_back = alg_bytes > L2_BYTES
    t_wall = time.time()
    if back_to_back:
        ev[0][0].record()
        for k in range(K):
            run_step(run.cache, steps[Wm + k], out, topk=w.topk, mass=mass)
        ev[0][1].record()
    else:
        for k in range(K):
            flush.zero_()
            inp = steps[Wm + k]
            # no event between the two calls (append + evict, decode): each kernel
            # may start while the previous one finishes (programmatic dependent launch)
            ev[k][0].record()
            run_step(run.cache, inp, out, topk=w.topk, mass=mass)
            ev[k][1].record()
    torch.cuda.synchronize()
    t_wall = time.time() - t_wall
    barrier(world)
    clk = clocks.stop(str(torch.cuda.get_device_properties(dev).uuid)) if clocks is not None else None
    assert run.cache.status() == 0, "device status after the timed steps"
    if back_to_back:
        step_ms = [ev[0][0].elapsed_time(ev[0][1]) / K] * K
    else:
        step_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(K)]
    # the decode call alone, for its roofline: the same launch on the state the
    # timed steps left, L2 flushed before each
    dev_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
    last = steps[Wm + K - 1]
    for k in range(K):
        flush.zero_()
        dev_ev[k][0].record()
        run.cache.decode(last.seqs, last.q, topk=w.topk, out=out, mass=mass)
        dev_ev[k][1].record()
    torch.cuda.synchronize()
    dec_ms = [a.elapsed_time(b) for a, b in dev_ev]
    res = {"step_s": sum(step_ms) / 1000.0, "steps": K, "tokens": float(w.batch * K),
           "step_ms": step_ms, "dec_ms": dec_ms, "alg_bytes": alg_bytes, "live": live,
           "pages": pages, "clocks": clk, "wall_s": t_wall,
           "l2": L2_LARGER if back_to_back else L2_FLUSHED}
    if compaction:
        res["compaction"] = measure_compaction(w, run, last, out, mass, live, K, flush, dev)

    if e2e_steps:
        # end to end through host buffers (pinned), copies inside the timed
        # region; each step's inputs packed in one pinned buffer: one copy
        host = [PackedStep(steps[Wm + K + k], "cpu", pin=True).fill(steps[Wm + K + k])
                for k in range(e2e_steps)]
        mass_shape = mass.shape if w.topk else None
        res["e2e_steps"] = e2e_steps
        res["e2e_tokens"] = float(w.batch * e2e_steps)
        res["h2d"] = host[0].nbytes()
        res["d2h"] = out.numel() * 2 + (mass.numel() * 4 if w.topk else 0)
        if alg_bytes > L2_BYTES:
            # each step reads more than L2 holds, so the steps may run back to
            # back: step k + 1's inputs are copied in (and step k - 1's output
            # copied out) while step k computes -- two device input buffers,
            # two output buffers, a stream per direction; the timed region runs
            # from the first input copy to the last output copy
            dbufs = [PackedStep(steps[Wm + K], dev) for _ in range(2)]
            outs = [torch.empty_like(out) for _ in range(2)]
            masses = [torch.empty(mass_shape, dtype=torch.float32, device=dev) if w.topk else None
                      for _ in range(2)]
            out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
            mass_h = [torch.empty(mass_shape, dtype=torch.float32).pin_memory() if w.topk else None
                      for _ in range(2)]
            s_c = torch.cuda.current_stream(dev)
            s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
            ev_in = [torch.cuda.Event() for _ in range(e2e_steps)]
            ev_done = [torch.cuda.Event() for _ in range(e2e_steps)]
            ev_out = [torch.cuda.Event() for _ in range(e2e_steps)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            t0.record(s_in)
            for k in range(e2e_steps):
                b = k % 2
                if k >= 2:
                    s_in.wait_event(ev_done[k - 2])       # step k - 2 has read this buffer
                with torch.cuda.stream(s_in):
                    dbufs[b].buf.copy_(host[k].buf, non_blocking=True)
                ev_in[k].record(s_in)
                s_c.wait_event(ev_in[k])
                if k >= 2:
                    s_c.wait_event(ev_out[k - 2])         # step k - 2's output has left
                run_step(run.cache, dbufs[b].inputs, outs[b], topk=w.topk, mass=masses[b])
                ev_done[k].record(s_c)
                s_out.wait_event(ev_done[k])
                with torch.cuda.stream(s_out):
                    out_h[b].copy_(outs[b], non_blocking=True)
                    if w.topk:
                        mass_h[b].copy_(masses[b], non_blocking=True)
                ev_out[k].record(s_out)
            t1.record(s_out)
            torch.cuda.synchronize()
            res["e2e_s"] = t0.elapsed_time(t1) / 1000.0
            res["e2e_mode"] = ("copies overlapped with compute (double-buffered, a stream per "
                               "direction); no L2 flush: each step reads more than L2 holds")
        else:
            dbuf = PackedStep(steps[Wm + K], dev)  # device staging, overwritten by the copies
            out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
            mass_h = torch.empty(mass_shape, dtype=torch.float32).pin_memory() if w.topk else None
            e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(e2e_steps)]
            torch.cuda.synchronize()
            for k in range(e2e_steps):
                flush.zero_()
                e2e_ev[k][0].record()
                run_step_from_host(run.cache, host[k], dbuf, out, out_h, topk=w.topk,
                                   mass_dev=mass, mass_host=mass_h)
                e2e_ev[k][1].record()
            torch.cuda.synchronize()
            res["e2e_s"] = sum(a.elapsed_time(b) for a, b in e2e_ev) / 1000.0
            res["e2e_mode"] = "one step at a time, L2 flushed between steps (outside the events)"
        assert run.cache.status() == 0, "device status after the end-to-end steps"
    del run, steps
    torch.cuda.empty_cache()
    return res


def roofline_block(w, res):
    """Roofline of the decode call from its algorithmic bytes and event time."""
    dec_avg_s = sum(res["dec_ms"]) / len(res["dec_ms"]) / 1000.0
    achieved = res["alg_bytes"] / dec_avg_s / 1e9
    peak, peak_kind = peak_hbm_gbs()
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic_per_launch(w.name),
            "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)",
            "kernel": DECODE_KERNELS,
            "algorithmic_bytes_per_launch": res["alg_bytes"], "live_pages": res["pages"]}


DECODE_KERNELS = "decode call: decode_split_kernel + decode_combine_kernel"


def thinkv_arm(args, w, world, rank, local):
    import torch
    from mixed_precision_paged_thinkv_b200 import build as B
    from mixed_precision_paged_thinkv_b200 import workloads as W
    B.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    K, Wm = args.steps, args.warmup
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    # the raw nvidia-smi samples go to THINKV_CLOCK_LOG_DIR (default: the temp dir)
    clocks = ClockSampler(os.path.join(os.environ.get("THINKV_CLOCK_LOG_DIR", tempfile.gettempdir()),
                                       f"thinkv_clocks_rank{rank}.csv"))
    e2e_steps = max(3, min(K, 100))   # as many as the device-timed steps, up to 100
    res = measure_workload(w, K, Wm, dev, flush, e2e_steps=e2e_steps, clocks=clocks, world=world,
                           compaction=(world == 1))
    max_s, tokens = dist_max_sum(res["step_s"], res["tokens"], world, dev)
    value = tokens / max_s
    e2e_max, e2e_tok = dist_max_sum(res["e2e_s"], res["e2e_tokens"], world, dev)

    # the other budgeted configurations, same run (single-GPU runs only)
    per_config = {}
    if world == 1 and not args.no_per_config and w.name == DEFAULT_WORKLOAD:
        for name in PER_CONFIG:
            wc = W.get(name)
            Kc = max(3, min(K, 20))
            rc = measure_workload(wc, Kc, 3, dev, flush)
            dec = sum(rc["dec_ms"]) / len(rc["dec_ms"])
            per_config[name] = {
                "config": workload_config(wc, rc["live"], rc["l2"]),
                "steps": Kc, "warmup": 3,
                "ms_per_step": 1000.0 * rc["step_s"] / Kc,
                "value": rc["tokens"] / rc["step_s"], "unit": "tokens/s",
                "decode_ms": dec,
                "decode_kv_tokens_per_s": float(sum(rc["live"])) / (dec / 1000.0),
                "roofline": roofline_block(wc, rc)}

    result = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            r = time_oracle(w, steps=5, warmup=1, budget_s=20.0, gen_device=str(dev))
            cpu = {"value": r["value"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                   "sample": _oracle_sample_text(w, r), "cpu_model": cpu_model(),
                   "decode_tokens_per_s": r["decode_tokens_per_s"],
                   "decode_tokens_per_s_1thread": r["decode_tokens_per_s_1thread"],
                   "setup_replay_s": r["setup_s"]}
        dec = sum(res["dec_ms"]) / len(res["dec_ms"])
        result = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": K, "warmup": Wm, "ms_per_step": 1000.0 * max_s / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16",
            "dtype_detail": "8/4/2-bit integer codes dequantised into f16 mma operands, f32 accumulate",
            "data": "synthetic (seeded counter-hash normals, segment tags)",
            "config": workload_config(w, res["live"], res["l2"]),
            "decode_ms": dec,
            "decode_hbm_gbs": res["alg_bytes"] / (dec / 1000.0) / 1e9,
            "decode_kv_tokens_per_s": float(sum(res["live"])) / (dec / 1000.0),
            "roofline": roofline_block(w, res),
            "per_config": per_config or None,
            "compaction_baseline": res.get("compaction"),
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_tok / e2e_max, "unit": "tokens/s", "h2d_bytes_per_step": res["h2d"],
                    "d2h_bytes_per_step": res["d2h"], "steps": res["e2e_steps"],
                    "mode": res["e2e_mode"]},
            "gpu_launches": launches_per_step(w.batch) * K,
            "clocks": res["clocks"],
            "wall_s_timed_loop": res["wall_s"],
        }
    return result


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="thinkv", choices=["thinkv", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the chosen workload (skip the per_config block)")
    args = ap.parse_args()
    from mixed_precision_paged_thinkv_b200 import workloads as W
    w = W.get(args.workload)
    world, rank, local = dist_init()
    try:
        if args.impl == "reference":
            return reference_arm(args, w, world, rank)
        res = thinkv_arm(args, w, world, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
        return 0
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())

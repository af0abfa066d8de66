"""Test harness: the same schedule driven through the oracle, and comparisons
of the GPU cache (libthinkv) against the oracle.

Inputs for both sides come only from ``workloads`` (the shared seeded
generator); expected values come only from ``oracle``.
"""
from __future__ import annotations

import numpy as np

from oracle import oracle as O
from mixed_precision_paged_thinkv_b200 import workloads as W

from layout_decode import decode_blocks

PAGE = 16
TOL = 2e-3          # row-normalised max error of decode outputs vs the fp64 oracle
MASS_TOL = 2e-3     # absolute error of the top-k attention mass


class OracleRun:
    """The oracle replaying a workload schedule (mirror of runner.WorkloadRun)."""

    def __init__(self, w: W.Workload, geom: dict, extra: int = 0, bits=None):
        self.w = w
        self.sched = W.Schedule(w, extra)
        self.o = O.Oracle(w.num_q_heads, w.num_kv_heads, w.head_dim, w.group_size,
                          bits or w.bits, geom["max_seqs"], geom["max_blocks_per_seq"],
                          geom["pool_pages"])
        self.generated = self.sched.lengths.astype(np.int64).copy()
        self.all_seqs = np.arange(w.batch, dtype=np.int32)

    def append_call(self, call):
        k, v = W.call_kv(self.w, call, device="cpu")
        st = self.o.append(call.seqs, call.pos, call.tags, k, v)
        assert st == O.OK, st

    def evict_all(self):
        assert self.o.evict(self.all_seqs, self.sched.budgets(self.generated)) == O.OK

    def decode(self, step, topk=None, threads=8):
        q = W.q_values(self.w, step, device="cpu")
        return self.o.decode(self.all_seqs, q, topk=topk, threads=threads)

    def setup(self):
        for call in self.sched.prefill_calls():
            self.append_call(call)
        self.evict_all()
        post = self.sched.post_evict_call()
        if post is not None:
            self.append_call(post)
            self.generated += self.w.post_evict_append
        for _ in range(self.w.churn_steps):
            self.churn_step()

    def churn_step(self, decode=False, step=0, topk=None):
        call = self.sched.one_token_call(self.generated)
        self.append_call(call)
        self.generated += 1
        self.evict_all()
        if decode:
            return self.decode(step, topk)
        return None


# --------------------------------------------------------------------------- #
# comparisons
# --------------------------------------------------------------------------- #
def compare_state(g: dict, o: dict, ns: int):
    """Bit-exact comparison of the slot bookkeeping (returns nothing, asserts)."""
    assert np.array_equal(g["page_bump"], o["page_bump"]), (g["page_bump"], o["page_bump"])
    assert np.array_equal(g["num_blocks"], o["num_blocks"])
    assert np.array_equal(g["live_count"], o["live_count"])
    assert np.array_equal(g["num_live"], o["num_live"])
    assert np.array_equal(g["free_top"], o["free_top"])
    assert np.array_equal(g["fifo_head"], o["fifo_head"])
    assert np.array_equal(g["fifo_tail"], o["fifo_tail"])
    cap = g["fifo"].shape[2]
    for s in range(ns):
        nb = int(o["num_blocks"][s])
        assert np.array_equal(g["table"][s, :nb], o["table"][s, :nb]), f"table of seq {s}"
        nl = int(o["num_live"][s])
        assert np.array_equal(g["live_list"][s, :nl], o["live_list"][s, :nl]), f"live list {s}"
        assert np.array_equal(g["live_index"][s, :nb], o["live_index"][s, :nb]), f"live index {s}"
        for c in range(3):
            top = int(o["free_top"][s, c])
            assert np.array_equal(g["free_slots"][s, c, :top], o["free_slots"][s, c, :top]), \
                f"free stack seq {s} class {c}"
            h, t = int(o["fifo_head"][s, c]), int(o["fifo_tail"][s, c])
            idx = np.arange(h, t) % cap
            assert np.array_equal(g["fifo"][s, c, idx], o["fifo"][s, c, idx]), f"fifo {s} {c}"
    for c in range(3):
        assert np.array_equal(g["slot_pos"][c], o["slot_pos"][c]), f"slot_pos class {c}"


def live_slots(o_state: dict, ns: int):
    """[(seq, class, page, slot)] of every live token, from the oracle's table."""
    out = []
    for s in range(ns):
        nb = int(o_state["num_blocks"][s])
        for e in o_state["table"][s, :nb]:
            page, cls, mask = int(O.entry_page(e)), int(O.entry_class(e)), int(O.entry_mask(e))
            for sl in range(PAGE):
                if (mask >> sl) & 1:
                    out.append((s, cls, page, sl))
    return out


def compare_codes(cache, oracle: O.Oracle, o_state: dict, ns: int, max_pages: int = None):
    """Codes and params of every live slot, bit for bit."""
    H, d, G = cache.H, cache.d, cache.G
    slots = live_slots(o_state, ns)
    by_class = {0: [], 1: [], 2: []}
    for (s, c, page, sl) in slots:
        by_class[c].append((page, sl))
    for c in range(3):
        if not by_class[c]:
            continue
        b = cache.bits[c]
        pages = np.array(sorted({p for p, _ in by_class[c]}))
        if max_pages is not None and len(pages) > max_pages:
            pages = np.random.default_rng(c).choice(pages, size=max_pages, replace=False)
        pool = cache.pool_bytes(c)[pages]                 # [np, H, phb]
        kc, vc, kp, vp = decode_blocks(pool, d, G, b)      # [np, H, 16, d] ...
        ocodes = oracle.codes(c)[pages]                    # [np, H, 2, 16, d]
        oparams = oracle.params(c)
        pidx = {int(p): i for i, p in enumerate(pages)}
        sel = [(pidx[p], sl) for (p, sl) in by_class[c] if p in pidx]
        pi = np.array([x[0] for x in sel])
        si = np.array([x[1] for x in sel])
        assert np.array_equal(kc[pi, :, si], ocodes[pi, :, 0, si]), f"K codes class {c}"
        assert np.array_equal(vc[pi, :, si], ocodes[pi, :, 1, si]), f"V codes class {c}"
        if b < 16:
            op = oparams[pages]
            assert np.array_equal(kp[pi, :, si], op[pi, :, 0, si]), f"K params class {c}"
            assert np.array_equal(vp[pi, :, si], op[pi, :, 1, si]), f"V params class {c}"


def attn_error(gpu_out: np.ndarray, ref: np.ndarray) -> float:
    """max over (sequence, head) rows of ||o - r||_inf / ||r||_inf (rows with r == 0: abs)."""
    g = gpu_out.astype(np.float64).reshape(-1, ref.shape[-1])
    r = ref.reshape(-1, ref.shape[-1])
    num = np.abs(g - r).max(axis=1)
    den = np.abs(r).max(axis=1)
    err = np.where(den > 0, num / np.where(den > 0, den, 1), num)
    return float(err.max()) if err.size else 0.0

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
                          geom["pool_pages"], fmt=w.fmt)
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


# --------------------------------------------------------------------------- #
# full-size checks on sampled sequences
# --------------------------------------------------------------------------- #
class OracleSubset:
    """The oracle replaying only some sequences of a workload.

    Sequences never interact except through the numbering of pages, so each
    sampled sequence's live set, codes and attention output equal those of a
    run over the whole batch.  Oracle sequence j stands for workload sequence
    seqs[j]; inputs come from the shared generator keyed by the original id."""

    def __init__(self, w: W.Workload, seqs, extra: int = 0, gen_device: str = "cuda"):
        import math
        self.w = w
        self.seqs = [int(s) for s in seqs]
        self.sched = W.Schedule(w, extra)
        self.gen_device = gen_device
        pool, mb = [0, 0, 0], 1
        for s in self.seqs:
            cnt = np.bincount(self.sched.tags(s), minlength=3)
            pages = [int(math.ceil(int(cnt[c]) / 16)) for c in range(3)]
            for c in range(3):
                pool[c] += pages[c]
            mb = max(mb, sum(pages))
        self.o = O.Oracle(w.num_q_heads, w.num_kv_heads, w.head_dim, w.group_size, w.bits,
                          len(self.seqs), mb, [max(1, p) for p in pool], fmt=w.fmt)
        self.generated = self.sched.lengths[self.seqs].astype(np.int64).copy()

    def _append(self, runs):
        """runs: [(j, pos0, count)] in call order (j = oracle sequence index)."""
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

    def _evict(self):
        b = self.sched.budgets(self.generated)
        assert self.o.evict(np.arange(len(self.seqs), dtype=np.int32), b) == O.OK

    def setup(self, churn: bool = True):
        where = {s: j for j, s in enumerate(self.seqs)}
        for call in self.sched.prefill_calls():
            self._append([(where[s], p0, c) for (s, p0, c) in call.runs if s in where])
        self._evict()
        if self.w.post_evict_append:
            n = self.w.post_evict_append
            self._append([(j, int(self.generated[j]), n) for j in range(len(self.seqs))])
            self.generated += n
        if churn:
            for _ in range(self.w.churn_steps):
                self.churn_step()

    def churn_step(self):
        self._append([(j, int(self.generated[j]), 1) for j in range(len(self.seqs))])
        self.generated += 1
        self._evict()

    def decode(self, step, topk=None):
        q = W.q_values(self.w, step, device="cpu")[self.seqs]
        return self.o.decode(np.arange(len(self.seqs), dtype=np.int32), q, topk=topk, threads=8)

    def live_by_pos(self, j):
        st = self.o.state()
        out = {}
        nb = int(st["num_blocks"][j])
        for e in st["table"][j, :nb]:
            page, cls, mask = int(O.entry_page(e)), int(O.entry_class(e)), int(O.entry_mask(e))
            for sl in range(PAGE):
                if (mask >> sl) & 1:
                    out[int(st["slot_pos"][cls][page, sl])] = (cls, page, sl)
        return out


def gpu_live_by_pos(snap, s):
    """pos -> (class, page, slot) of every live token of GPU sequence s."""
    out = {}
    nb = int(snap["num_blocks"][s])
    for e in snap["table"][s, :nb]:
        page, cls, mask = int(O.entry_page(e)), int(O.entry_class(e)), int(O.entry_mask(e))
        for sl in range(PAGE):
            if (mask >> sl) & 1:
                out[int(snap["slot_pos"][cls][page, sl])] = (cls, page, sl)
    return out


def _gpu_blocks(cache, c, pages):
    """Page-head blocks [len(pages), Hkv, phb] of class c, copied from the GPU."""
    import torch
    phb = cache.page_head_bytes(c)
    pool = cache.buf["pool_" + "RET"[c]].view(cache.pool_pages[c], cache.H, phb)
    idx = torch.as_tensor(np.asarray(pages, dtype=np.int64), device=pool.device)
    return pool[idx].cpu().numpy()


def compare_codes_by_pos(cache, gl: dict, oracle: O.Oracle, ol: dict):
    """Codes and params of every live token, matched by position, bit for bit."""
    d, G = cache.d, cache.G
    for c in range(3):
        poss = [p for p in gl if gl[p][0] == c]
        if not poss:
            continue
        b = cache.bits[c]
        gpages = [gl[p][1] for p in poss]
        gslots = np.array([gl[p][2] for p in poss])
        kc, vc, kp, vp = decode_blocks(_gpu_blocks(cache, c, gpages), d, G, b)
        n = np.arange(len(poss))
        opages = np.array([ol[p][1] for p in poss])
        oslots = np.array([ol[p][2] for p in poss])
        ocodes = oracle.codes(c)
        assert np.array_equal(kc[n, :, gslots], ocodes[opages, :, 0, oslots]), f"K codes class {c}"
        assert np.array_equal(vc[n, :, gslots], ocodes[opages, :, 1, oslots]), f"V codes class {c}"
        if b < 16:
            op = oracle.params(c)
            assert np.array_equal(kp[n, :, gslots], op[opages, :, 0, oslots]), f"K params class {c}"
            assert np.array_equal(vp[n, :, gslots], op[opages, :, 1, oslots]), f"V params class {c}"


def compare_seq_structure(g: dict, s: int, o: dict, j: int):
    """Bit-exact comparison of GPU sequence s with oracle sequence j, where the
    two runs number pool pages differently (the oracle replays a subset of the
    batch).  Everything the state holds per sequence is in per-sequence terms
    (table entry indices, slot ids entry*16 + slot, counters) and must match
    exactly; page ids are compared through the entry -> page map each side's
    table defines, which must be one-to-one on (class, page)."""
    for key in ("num_blocks", "live_count", "num_live"):
        assert int(g[key][s]) == int(o[key][j]), f"{key} of seq {s}"
    for key in ("free_top", "fifo_head", "fifo_tail"):
        assert np.array_equal(g[key][s], o[key][j]), f"{key} of seq {s}"
    nb = int(o["num_blocks"][j])
    gt, ot = g["table"][s, :nb], o["table"][j, :nb]
    assert np.array_equal(O.entry_class(gt), O.entry_class(ot)), f"entry classes of seq {s}"
    assert np.array_equal(O.entry_mask(gt), O.entry_mask(ot)), f"entry masks of seq {s}"
    gp, op = O.entry_page(gt).astype(np.int64), O.entry_page(ot).astype(np.int64)
    # page ids number each class pool separately: (class, page) is the key
    gkey = (O.entry_class(gt).astype(np.int64) << 32) | gp
    assert len(set(gkey.tolist())) == nb, f"GPU pages of seq {s} repeat"
    # slot positions of every slot of every entry, through the page map
    for c in range(3):
        sel = np.flatnonzero(O.entry_class(ot) == c)
        if sel.size:
            gsp = g["slot_pos"][c][gp[sel]]
            osp = o["slot_pos"][c][op[sel]]
            assert np.array_equal(gsp, osp), f"slot_pos of seq {s} class {c}"
    cap = g["fifo"].shape[2]
    for c in range(3):
        top = int(o["free_top"][j, c])
        assert np.array_equal(g["free_slots"][s, c, :top], o["free_slots"][j, c, :top]), \
            f"free stack of seq {s} class {c}"
        h, t = int(o["fifo_head"][j, c]), int(o["fifo_tail"][j, c])
        idx = np.arange(h, t) % cap
        assert np.array_equal(g["fifo"][s, c, idx], o["fifo"][j, c, idx]), f"fifo of seq {s} class {c}"
    nl = int(o["num_live"][j])
    gl, ol = g["live_list"][s, :nl], o["live_list"][j, :nl]
    assert np.array_equal(O.live_entry(gl), O.live_entry(ol)), f"live list order of seq {s}"
    assert np.array_equal(O.entry_class(gl), O.entry_class(ol)), f"live list classes of seq {s}"
    assert np.array_equal(O.entry_page(gl).astype(np.int64), gp[O.live_entry(gl)]), \
        f"live list pages of seq {s}"
    assert np.array_equal(g["live_index"][s, :nb], o["live_index"][j, :nb]), f"live index of seq {s}"


def check_slot_invariants(snap, ns):
    """Free-slot invariants of every sequence (no oracle needed): per (sequence,
    class) the allocated slots are exactly the live ones plus the free-stack
    ones, each once; live_count and num_live agree with the masks; the live
    list and its index invert each other; the FIFO window holds the live slots."""
    cap = snap["fifo"].shape[2]
    for s in range(ns):
        nb = int(snap["num_blocks"][s])
        ents = snap["table"][s, :nb]
        cls = O.entry_class(ents)
        masks = O.entry_mask(ents)
        bits = ((masks[:, None] >> np.arange(PAGE)[None, :]) & 1).astype(bool)
        assert int(bits.sum()) == int(snap["live_count"][s])
        nl = int(snap["num_live"][s])
        assert nl == int((masks != 0).sum())
        lst = O.live_entry(snap["live_list"][s, :nl])
        assert np.array_equal(snap["live_index"][s, lst], np.arange(nl))
        for c in range(3):
            mark = np.zeros(nb * PAGE, dtype=np.int32)
            own = np.repeat(cls == c, PAGE)
            live_ids = np.flatnonzero(bits.reshape(-1) & own)
            mark[live_ids] += 1
            top = int(snap["free_top"][s, c])
            free = snap["free_slots"][s, c, :top]
            assert free.size == 0 or (free.min() >= 0 and free.max() < nb * PAGE)
            np.add.at(mark, free, 1)
            assert np.array_equal(mark, own.astype(np.int32)), f"free/live slots, seq {s} class {c}"
            h, t = int(snap["fifo_head"][s, c]), int(snap["fifo_tail"][s, c])
            win = snap["fifo"][s, c, np.arange(h, t) % cap]
            win = win[win >= 0]                            # -1: tombstones of TBE evictions
            assert np.array_equal(np.sort(win), live_ids)

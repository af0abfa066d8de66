"""The sampled full-size GPU checks replay only a few sequences through the
oracle.  That is sound because sequences share nothing but the numbering of
pool pages: here, on a reduced churn workload, the oracle replaying a subset
gives, for every sampled sequence, the same live positions and classes, the
same codes and params per position, and the same decode rows and top-k masses
as the oracle replaying the whole batch."""
import numpy as np

from oracle import oracle as O
from mixed_precision_paged_thinkv_b200 import workloads as W
from mixed_precision_paged_thinkv_b200.runner import geometry

import harness as Hn


def _by_pos(state, s):
    out = {}
    nb = int(state["num_blocks"][s])
    for e in state["table"][s, :nb]:
        page, cls, mask = int(O.entry_page(e)), int(O.entry_class(e)), int(O.entry_mask(e))
        for sl in range(Hn.PAGE):
            if (mask >> sl) & 1:
                out[int(state["slot_pos"][cls][page, sl])] = (cls, page, sl)
    return out


def test_subset_replay_equals_full_replay():
    w = W.scaled(W.WORKLOADS["churn"], batch=6, lengths=("loguniform", 300, 2500),
                 churn_steps=12, topk=8, budget=("frac", 0.1))
    sched = W.Schedule(w, 0)
    full = Hn.OracleRun(w, geometry(w, sched), extra=0)
    full.setup()
    seqs = [1, 4, 5]
    sub = Hn.OracleSubset(w, seqs, extra=0, gen_device="cpu")
    sub.setup()
    fs = full.o.state()
    ss = sub.o.state()
    Hn.check_slot_invariants(fs, w.batch)
    Hn.check_slot_invariants(ss, len(seqs))
    for j, s in enumerate(seqs):
        # the whole per-sequence state, through the entry -> page map
        Hn.compare_seq_structure(fs, s, ss, j)
        a, b = _by_pos(fs, s), sub.live_by_pos(j)
        assert sorted(a) == sorted(b)
        for c in range(3):
            pos = [p for p in a if a[p][0] == c]
            assert all(b[p][0] == c for p in pos)
            if not pos:
                continue
            fa = full.o.codes(c)[[a[p][1] for p in pos], :, :, [a[p][2] for p in pos]]
            fb = sub.o.codes(c)[[b[p][1] for p in pos], :, :, [b[p][2] for p in pos]]
            assert np.array_equal(fa, fb)
            pa = full.o.params(c)[[a[p][1] for p in pos], :, :, [a[p][2] for p in pos]]
            pb = sub.o.params(c)[[b[p][1] for p in pos], :, :, [b[p][2] for p in pos]]
            assert np.array_equal(pa, pb)
    ro, rm = full.decode(3, topk=w.topk)
    so, sm = sub.decode(3, topk=w.topk)
    assert np.array_equal(ro[seqs], so)
    assert np.array_equal(rm[seqs], sm)


def test_slot_invariants_catch_a_lost_slot():
    w = W.scaled(W.WORKLOADS["churn"], batch=2, lengths=("fixed", 400), churn_steps=3)
    sub = Hn.OracleSubset(w, [0, 1], extra=0, gen_device="cpu")
    sub.setup()
    st = sub.o.state()
    Hn.check_slot_invariants(st, 2)
    c = int(np.argmax(st["free_top"][1]))
    assert st["free_top"][1, c] > 0
    st["free_top"][1, c] -= 1            # one free slot dropped from the stack
    try:
        Hn.check_slot_invariants(st, 2)
    except AssertionError:
        return
    raise AssertionError("a slot missing from the free stack went unnoticed")


def test_structure_comparison_catches_planted_differences():
    """compare_seq_structure (used on the full-size GPU states) must notice a
    swapped FIFO pair, a flipped mask bit, a reordered free stack, a moved
    live-list entry and a wrong slot position."""
    import copy
    w = W.scaled(W.WORKLOADS["churn"], batch=3, lengths=("fixed", 700), churn_steps=5,
                 budget=("frac", 0.2))
    sched = W.Schedule(w, 0)
    full = Hn.OracleRun(w, geometry(w, sched), extra=0)
    full.setup()
    sub = Hn.OracleSubset(w, [2], extra=0, gen_device="cpu")
    sub.setup()
    fs, ss = full.o.state(), sub.o.state()
    Hn.compare_seq_structure(fs, 2, ss, 0)
    cap = ss["fifo"].shape[2]

    def plant(edit):
        st = copy.deepcopy(ss)
        edit(st)
        try:
            Hn.compare_seq_structure(fs, 2, st, 0)
        except AssertionError:
            return
        raise AssertionError("a planted difference went unnoticed")

    c = int(np.argmax(ss["fifo_tail"][0] - ss["fifo_head"][0]))
    h = int(ss["fifo_head"][0, c])

    def swap_fifo(st):
        a, b = h % cap, (h + 1) % cap
        st["fifo"][0, c, [a, b]] = st["fifo"][0, c, [b, a]]
    plant(swap_fifo)

    def flip_mask(st):
        st["table"][0, 0] ^= np.uint64(1 << 48)
    plant(flip_mask)

    cf = int(np.argmax(ss["free_top"][0]))

    def reorder_stack(st):
        st["free_slots"][0, cf, [0, 1]] = st["free_slots"][0, cf, [1, 0]]
    assert ss["free_top"][0, cf] >= 2
    plant(reorder_stack)

    def move_live(st):
        st["live_list"][0, [0, 1]] = st["live_list"][0, [1, 0]]
    assert ss["num_live"][0] >= 2
    plant(move_live)

    def wrong_pos(st):
        e = st["table"][0, 0]
        cls, page = int(O.entry_class(e)), int(O.entry_page(e))
        st["slot_pos"][cls][page, 3] += 1
    plant(wrong_pos)

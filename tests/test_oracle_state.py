"""Pins of the oracle's slot bookkeeping (continuous-thinking slot reuse, CT).

* a scripted history worked by hand (tests/golden/slots_example.json);
* random histories against an independent set model: which tokens are live
  after every operation, and the structural invariants of the tables;
* all-or-nothing error behaviour.
"""
import json
import os

import numpy as np
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "slots_example.json")
PAGE = 16


def _oracle(L):
    return O.Oracle(L["num_q_heads"], L["num_kv_heads"], L["head_dim"], L["group_size"],
                    L["bits"], L["max_seqs"], L["max_blocks_per_seq"], L["pool_pages"])


def _kv(n, H, d, seed=0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, H, d)).astype(np.float16),
            rng.standard_normal((n, H, d)).astype(np.float16))


def _table(st, s):
    t = st["table"][s, :st["num_blocks"][s]]
    return [[int(O.entry_page(e)), int(O.entry_class(e)), int(O.entry_mask(e))] for e in t]


def _free(st, s, c):
    return st["free_slots"][s, c, :st["free_top"][s, c]].tolist()


def _fifo(st, s, c):
    cap = st["fifo"].shape[2]
    h, t = st["fifo_head"][s, c], st["fifo_tail"][s, c]
    return [int(st["fifo"][s, c, i % cap]) for i in range(h, t)]


def test_scripted_history_worked_by_hand():
    g = json.load(open(GOLDEN))
    L = g["layout"]
    o = _oracle(L)
    H, d = L["num_kv_heads"], L["head_dim"]
    k, v = _kv(20, H, d)
    assert o.append([0] * 20, list(range(20)), [0] * 20, k, v) == O.OK
    k, v = _kv(3, H, d, 1)
    assert o.append([1, 1, 1], [0, 1, 2], [2, 2, 1], k, v) == O.OK
    st = o.state()
    e = g["after_op2"]
    assert st["page_bump"].tolist() == e["page_bump"]
    assert st["num_blocks"].tolist() == e["num_blocks"]
    assert _table(st, 0) == e["table_seq0"]
    assert _table(st, 1) == e["table_seq1"]
    assert _free(st, 0, 0) == e["free_seq0_R"]
    assert _free(st, 1, 2) == e["free_seq1_T"]
    assert _free(st, 1, 1) == e["free_seq1_E"]
    assert _fifo(st, 0, 0) == e["fifo_seq0_R"]
    assert _fifo(st, 1, 2) == e["fifo_seq1_T"]
    assert _fifo(st, 1, 1) == e["fifo_seq1_E"]
    assert [O.live_entry(st["live_list"][s, :st["num_live"][s]]).tolist() for s in range(2)] == e["live_list"]
    # descriptors carry the page and class of their entry
    for s in range(2):
        for x in st["live_list"][s, :st["num_live"][s]]:
            ent = st["table"][s, int(O.live_entry(x))]
            assert int(O.entry_page(x)) == int(O.entry_page(ent))
            assert int(O.entry_class(x)) == int(O.entry_class(ent))
    assert st["live_count"].tolist() == e["live_count"]
    assert st["slot_pos"][0][1].tolist() == e["slot_pos_R_page1"]

    assert o.evict([0], [8]) == O.OK
    st = o.state()
    e = g["after_op3"]
    assert [m for (_, _, m) in _table(st, 0)] == e["masks_seq0"]
    assert _free(st, 0, 0) == e["free_seq0_R"]
    assert _fifo(st, 0, 0) == e["fifo_window_seq0_R"]
    assert st["live_count"].tolist() == e["live_count"]
    assert st["slot_pos"][0][0].tolist() == e["slot_pos_R_page0"]

    k, v = _kv(2, H, d, 2)
    assert o.append([0, 0], [20, 21], [0, 0], k, v) == O.OK
    st = o.state()
    e = g["after_op4"]
    assert [m for (_, _, m) in _table(st, 0)] == e["masks_seq0"]
    assert st["slot_pos"][0][0].tolist() == e["slot_pos_R_page0"]
    assert _fifo(st, 0, 0) == e["fifo_window_seq0_R"]
    assert int(st["free_top"][0, 0]) == e["free_top_seq0_R"]

    assert o.evict([0], [0]) == O.OK
    st = o.state()
    e = g["after_op5"]
    assert [m for (_, _, m) in _table(st, 0)] == e["masks_seq0"]
    assert st["num_live"].tolist() == e["num_live"]
    assert st["live_count"].tolist() == e["live_count"]
    assert _free(st, 0, 0) == e["free_seq0_R"]
    q = np.ones((1, 1, d), dtype=np.float16)
    out, mass = o.decode([0], q, topk=4)
    assert not out.any() and not mass.any()


# --------------------------------------------------------------------------- #
# independent model: the live set is a set of (seq, pos); eviction removes the
# oldest live tokens of the first non-empty class in the order T, E, R
# --------------------------------------------------------------------------- #
class SetModel:
    def __init__(self, ns):
        self.live = [dict() for _ in range(ns)]   # pos -> class

    def append(self, seqs, pos, tags):
        for s, p, c in zip(seqs, pos, tags):
            self.live[s][int(p)] = int(c)

    def evict(self, seqs, budgets, order=(2, 1, 0)):
        for s, b in zip(seqs, budgets):
            n = len(self.live[s]) - b
            for _ in range(max(0, n)):
                for c in order:
                    cand = sorted(p for p, cc in self.live[s].items() if cc == c)
                    if cand:
                        del self.live[s][cand[0]]
                        break


def _check_invariants(o, st, model, ns):
    cap = o.max_blocks * PAGE
    owner = {}
    for s in range(ns):
        nb = st["num_blocks"][s]
        ents = st["table"][s, :nb]
        pages, classes, masks = O.entry_page(ents), O.entry_class(ents), O.entry_mask(ents)
        # each page belongs to exactly one sequence
        for p, c in zip(pages, classes):
            assert (int(c), int(p)) not in owner
            owner[(int(c), int(p))] = s
        # live tokens = popcount of masks = live_count = model
        pop = sum(bin(int(m)).count("1") for m in masks)
        assert pop == st["live_count"][s] == len(model.live[s])
        live_pos = {}
        for e, (p, c, m) in enumerate(zip(pages, classes, masks)):
            for sl in range(PAGE):
                sp = st["slot_pos"][int(c)][int(p), sl]
                if (int(m) >> sl) & 1:
                    live_pos[int(sp)] = int(c)
                else:
                    assert sp == -1
        assert live_pos == model.live[s]
        # live list = entries with a non-zero mask; live_index inverts it
        nl = st["num_live"][s]
        desc = st["live_list"][s, :nl]
        lst = O.live_entry(desc)
        assert sorted(lst.tolist()) == [e for e in range(nb) if masks[e]]
        assert np.array_equal(O.entry_page(desc), pages[lst])
        assert np.array_equal(O.entry_class(desc), classes[lst])
        for i, e in enumerate(lst):
            assert st["live_index"][s, e] == i
        for e in range(nb):
            if not masks[e]:
                assert st["live_index"][s, e] == -1
        for c in range(3):
            ids_c = {e * PAGE + sl for e in range(nb) if classes[e] == c for sl in range(PAGE)}
            live_c = {e * PAGE + sl for e in range(nb) if classes[e] == c
                      for sl in range(PAGE) if (int(masks[e]) >> sl) & 1}
            free_c = st["free_slots"][s, c, :st["free_top"][s, c]].tolist()
            # allocated slots of the class = live + free, disjoint, no duplicates
            assert len(free_c) == len(set(free_c))
            assert set(free_c).isdisjoint(live_c)
            assert set(free_c) | live_c == ids_c
            # the FIFO window holds exactly the live slots of the class, in position order
            h, t = st["fifo_head"][s, c], st["fifo_tail"][s, c]
            win = [int(st["fifo"][s, c, i % cap]) for i in range(h, t)]
            assert set(win) == live_c and len(win) == len(live_c)
            posw = []
            for ts in win:
                e, sl = divmod(ts, PAGE)
                posw.append(int(st["slot_pos"][c][int(pages[e]), sl]))
            assert posw == sorted(posw) and len(set(posw)) == len(posw)


@pytest.mark.parametrize("seed", range(6))
def test_random_histories_against_set_model(seed):
    rng = np.random.default_rng(seed)
    ns, H, d = 3, 1, 32
    o = O.Oracle(2, H, d, 32, (8, 4, 2), ns, 40, (60, 60, 60))
    model = SetModel(ns)
    nextpos = [0] * ns
    for op in range(200):
        if rng.random() < 0.6:
            seqs = rng.permutation(ns)[:rng.integers(1, ns + 1)]
            S, P, T = [], [], []
            for s in seqs:
                c = int(rng.integers(1, 12))
                for _ in range(c):
                    S.append(int(s)); P.append(nextpos[s]); T.append(int(rng.choice(3, p=[.3, .5, .2])))
                    nextpos[s] += 1
            k, v = _kv(len(S), H, d, op)
            st = o.append(S, P, T, k, v)
            assert st == O.OK
            model.append(S, P, T)
        else:
            seqs = rng.permutation(ns)[:rng.integers(1, ns + 1)]
            budgets = [int(rng.integers(0, 30)) for _ in seqs]
            order = None if rng.random() < 0.7 else list(rng.permutation(3))
            assert o.evict(seqs, budgets, order) == O.OK
            model.evict(seqs, budgets, tuple(order) if order is not None else (2, 1, 0))
        _check_invariants(o, o.state(), model, ns)


def test_errors_are_all_or_nothing():
    H, d = 1, 32
    o = O.Oracle(1, H, d, 32, (8, 4, 2), 2, 3, (2, 1, 1))
    k, v = _kv(40, H, d)
    before = o.state()
    # 40 R tokens need 3 R pages; the pool has 2
    assert o.append([0] * 40, list(range(40)), [0] * 40, k, v) == O.ERR_OUT_OF_PAGES
    after = o.state()
    for key in ("num_blocks", "free_top", "fifo_tail", "live_count", "page_bump"):
        assert np.array_equal(before[key], after[key])
    # tokens of one sequence split into two runs -> invalid
    assert o.append([0, 1, 0], [0, 0, 1], [0, 0, 0], k[:3], v[:3]) == O.ERR_INVALID
    # positions not ascending inside a run -> invalid
    assert o.append([0, 0], [5, 4], [0, 0], k[:2], v[:2]) == O.ERR_INVALID
    # bad tag / bad sequence -> invalid
    assert o.append([0], [0], [3], k[:1], v[:1]) == O.ERR_INVALID
    assert o.append([2], [0], [0], k[:1], v[:1]) == O.ERR_INVALID
    # table full: 3 entries per sequence, E and T pools have 1 page each
    assert o.append([0] * 17, list(range(17)), [1] * 17, k[:17], v[:17]) == O.ERR_OUT_OF_PAGES
    # evict: duplicate sequences, negative budget, bad order -> invalid; budget > live -> no-op
    assert o.evict([0, 0], [1, 1]) == O.ERR_INVALID
    assert o.evict([0], [-1]) == O.ERR_INVALID
    assert o.evict([0], [1], [0, 0, 1]) == O.ERR_INVALID
    assert o.append([0] * 5, list(range(5)), [0] * 5, k[:5], v[:5]) == O.OK
    assert o.evict([0], [100]) == O.OK
    assert o.state()["live_count"][0] == 5


def test_out_of_blocks():
    H, d = 1, 32
    o = O.Oracle(1, H, d, 32, (8, 4, 2), 1, 2, (8, 8, 8))
    k, v = _kv(3, H, d)
    # three classes need three table entries; only two fit
    assert o.append([0, 0, 0], [0, 1, 2], [0, 1, 2], k, v) == O.ERR_OUT_OF_BLOCKS
    assert o.append([0, 0], [0, 1], [0, 1], k[:2], v[:2]) == O.OK

"""Pins of the oracle's TBE (segment-level eviction on Transition thoughts)
and of its tombstone-aware budget eviction:

- a scripted history worked by hand into the expected live sets, segment
  records, FIFO windows (with tombstones) and free stacks
  (tests/golden/tbe_example.json), with the appends in one call and one token
  per call;
- an independent brute-force model that knows nothing of FIFOs, slots or
  tombstones -- per sequence, the live positions of each same-tag run -- on
  random histories with random call splits, budget evictions, schedules and
  safety nets;
- the slot invariants (allocated = live + free, FIFO windows = live slots plus
  tombstones) after every operation.
"""
import json
import os

import numpy as np
import pytest

from oracle import oracle as O

import harness as Hn

HERE = os.path.dirname(os.path.abspath(__file__))
CLS = {"R": 0, "E": 1, "T": 2}


def _kv(n, H, d, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, H, d)).astype(np.float16),
            rng.standard_normal((n, H, d)).astype(np.float16))


def _live_by_class(st, s=0):
    out = {0: [], 1: [], 2: []}
    for e in st["table"][s, :int(st["num_blocks"][s])]:
        c, page, mask = int(O.entry_class(e)), int(O.entry_page(e)), int(O.entry_mask(e))
        for sl in range(16):
            if (mask >> sl) & 1:
                out[c].append(int(st["slot_pos"][c][page, sl]))
    return {c: sorted(v) for c, v in out.items()}


def _fifo_positions(st, s, c, pos_of_slot):
    cap = st["fifo"].shape[2]
    h, t = int(st["fifo_head"][s, c]), int(st["fifo_tail"][s, c])
    win = st["fifo"][s, c, np.arange(h, t) % cap]
    return h, t, [-1 if x < 0 else pos_of_slot[int(x)] for x in win]


@pytest.mark.parametrize("per_token", [False, True])
def test_hand_worked_tbe_history(per_token):
    g = json.load(open(os.path.join(HERE, "golden", "tbe_example.json")))
    geo = g["geometry"]
    o = O.Oracle(geo["num_q_heads"], geo["num_kv_heads"], geo["head_dim"], geo["group_size"],
                 geo["bits"], geo["max_seqs"], geo["max_blocks_per_seq"], geo["pool_pages"])
    tags = np.array([CLS[t] for t in g["tags"]], dtype=np.uint8)
    k, v = _kv(len(tags), geo["num_kv_heads"], geo["head_dim"], 0)
    pos_of_slot = {}                   # (entry*16 + slot) -> position, as appended
    for step in g["steps"]:
        if step["op"] == "append+tbe":
            a, b = step["positions"]
            calls = [(p, p + 1) for p in range(a, b)] if per_token else [(a, b)]
            for (p0, p1) in calls:
                seq = np.zeros(p1 - p0, np.int32)
                pos = np.arange(p0, p1, dtype=np.int32)
                assert o.append(seq, pos, tags[p0:p1], k[p0:p1], v[p0:p1]) == O.OK
                st = o.state()
                for p in range(p0, p1):       # where each new token went, before any eviction
                    c = int(tags[p])
                    h, t = int(st["fifo_head"][0, c]), int(st["fifo_tail"][0, c])
                    cap = st["fifo"].shape[2]
                    win = st["fifo"][0, c, np.arange(h, t) % cap]
                    for x in win:
                        if x >= 0:
                            e, sl = int(x) // 16, int(x) % 16
                            page = int(O.entry_page(st["table"][0, e]))
                            if int(st["slot_pos"][c][page, sl]) == p:
                                pos_of_slot[int(x)] = p
                assert o.tbe(seq, pos, tags[p0:p1], t_min=g["t_min"], schedule=g["schedule"]) == O.OK
        else:
            assert o.evict(np.zeros(1, np.int32), np.array([step["budget"]], np.int32)) == O.OK
        st = o.state()
        Hn.check_slot_invariants(st, 1)
        live = _live_by_class(st)
        assert {n: live[c] for n, c in CLS.items()} == step["live"], (step["op"], live)
        assert int(st["live_count"][0]) == step["live_count"]
        if "seg" in step:
            ns = int(st["nseg"][0])
            assert st["seg"][0, :ns].tolist() == step["seg"]
        for n, c in CLS.items():
            h, t, win = _fifo_positions(st, 0, c, pos_of_slot)
            eh, et, ewin = step["fifo"][n]
            assert (h, t, win) == (eh, et, ewin), (step["op"], n, (h, t, win))
        if not per_token and "free_one_call" in step:
            for n, c in CLS.items():
                top = int(st["free_top"][0, c])
                assert st["free_slots"][0, c, :top].tolist() == step["free_one_call"][n], n


# --------------------------------------------------------------------------- #
# independent model: live positions per same-tag run, nothing else
# --------------------------------------------------------------------------- #
class Model:
    def __init__(self, schedule, t_min):
        self.schedule, self.t_min = list(schedule), t_min
        self.segs = {}      # seq -> [[cls, level, [live positions ascending]]]
        self.tag_of = {}

    def append_tbe(self, seqs, poss, tags):
        for s, p, c in zip(seqs.tolist(), poss.tolist(), tags.tolist()):
            self.tag_of[(s, p)] = c
            segs = self.segs.setdefault(s, [])
            if segs and segs[-1][0] == c:
                segs[-1][2].append(p)
                continue
            segs.append([c, 0, [p]])
            if c == 2:
                self.event(segs, len(segs) - 1)

    def event(self, segs, e):
        net = self.t_min
        keep_t = {}
        for j in range(e - 1, -1, -1):
            if segs[j][0] == 2:
                k = min(len(segs[j][2]), net)
                keep_t[j] = k
                net -= k
        for j in range(e):
            c, lvl, live = segs[j]
            if c == 2:
                keep = keep_t[j]
            else:
                lvl = min(lvl + 1, 3)
                segs[j][1] = lvl
                keep = self.schedule[lvl - 1]
            if len(live) > keep:
                del live[:len(live) - keep]          # oldest go first

    def evict(self, s, budget, order=(2, 1, 0)):
        segs = self.segs.get(s, [])
        n = sum(len(g[2]) for g in segs) - budget
        for _ in range(max(0, n)):
            for c in order:
                cand = [(g[2][0], g) for g in segs if g[0] == c and g[2]]
                if cand:
                    p, g = min(cand, key=lambda x: x[0])
                    g[2].pop(0)
                    break

    def live(self, s):
        out = {0: [], 1: [], 2: []}
        for c, _, live in self.segs.get(s, []):
            out[c].extend(live)
        return {c: sorted(v) for c, v in out.items()}


@pytest.mark.parametrize("seed", range(12))
def test_tbe_against_position_model(seed):
    rng = np.random.default_rng(100 + seed)
    ns, L = 3, 700
    schedule = [int(x) for x in sorted(rng.integers(1, 12, 3), reverse=True)]
    t_min = int(rng.integers(0, 6))
    H, d = 1, 64
    tags = {}
    for s in range(ns):
        t = []
        while len(t) < L:
            t += [int(rng.choice(3, p=[0.35, 0.4, 0.25]))] * int(rng.integers(1, 9))
        tags[s] = np.array(t[:L], np.uint8)
    o = O.Oracle(4, H, d, 32, (8, 4, 2), ns, L // 16 * 3 + 8, (ns * L // 16 + 8,) * 3)
    m = Model(schedule, t_min)
    done = [0] * ns
    while min(done) < L:
        # one call: a run of random length for each sequence that has tokens left
        seqs, poss, tg = [], [], []
        for s in rng.permutation(ns).tolist():
            if done[s] >= L:
                continue
            cnt = int(min(L - done[s], rng.integers(1, 40)))
            seqs += [s] * cnt
            poss += list(range(done[s], done[s] + cnt))
            tg += tags[s][done[s]:done[s] + cnt].tolist()
            done[s] += cnt
        seqs, poss, tg = (np.array(seqs, np.int32), np.array(poss, np.int32), np.array(tg, np.uint8))
        k, v = _kv(len(seqs), H, d, int(rng.integers(1 << 30)))
        assert o.append(seqs, poss, tg, k, v) == O.OK
        assert o.tbe(seqs, poss, tg, t_min=t_min, schedule=schedule) == O.OK
        m.append_tbe(seqs, poss, tg)
        if rng.random() < 0.3:
            s = int(rng.integers(ns))
            live_now = sum(len(x) for x in m.live(s).values())
            b = int(rng.integers(0, live_now + 1))
            order = [int(x) for x in rng.permutation(3)]
            assert o.evict(np.array([s], np.int32), np.array([b], np.int32), order=order) == O.OK
            m.evict(s, b, order)
        st = o.state()
        Hn.check_slot_invariants(st, ns)
        for s in range(ns):
            assert _live_by_class(st, s) == m.live(s), (seed, s)
            assert int(st["live_count"][s]) == sum(len(x) for x in m.live(s).values())
    # the schedule's effect is visible: every ended R/E segment is within its retention
    st = o.state()
    for s in range(ns):
        segs = m.segs[s]
        for j, (c, lvl, live) in enumerate(segs):
            if c != 2 and lvl > 0:
                assert len(live) <= schedule[lvl - 1]


def test_tbe_rejects_bad_calls_and_changes_nothing():
    o = O.Oracle(2, 1, 64, 32, (8, 4, 2), 2, 4, (4, 4, 4))
    k, v = _kv(3, 1, 64, 1)
    seq = np.zeros(3, np.int32)
    pos = np.arange(3, dtype=np.int32)
    tag = np.array([0, 2, 0], np.uint8)
    assert o.append(seq, pos, tag, k, v) == O.OK
    before = o.state()
    assert o.tbe(seq, pos, tag, t_min=-1) == O.ERR_INVALID
    assert o.tbe(seq, pos, tag, schedule=[4, -1, 1]) == O.ERR_INVALID
    assert o.tbe(np.array([0, 1, 0], np.int32), pos, tag) == O.ERR_INVALID      # seq 0 in two runs
    assert o.tbe(seq, np.array([0, 2, 1], np.int32), tag) == O.ERR_INVALID      # positions not ascending
    assert o.tbe(seq, pos, np.array([0, 3, 0], np.uint8)) == O.ERR_INVALID      # tag > 2
    after = o.state()
    for key in before:
        if key == "slot_pos":
            assert all(np.array_equal(a, b) for a, b in zip(before[key], after[key]))
        else:
            assert np.array_equal(before[key], after[key]), key


def test_tbe_rejects_tokens_the_append_did_not_store():
    """Class counts that exceed what the FIFOs hold: the call did not follow
    an append of these tokens; rejected, nothing changes."""
    o = O.Oracle(2, 1, 64, 32, (8, 4, 2), 1, 4, (4, 4, 4))
    k, v = _kv(4, 1, 64, 2)
    seq = np.zeros(2, np.int32)
    assert o.append(seq, np.arange(2, dtype=np.int32), np.array([0, 0], np.uint8), k[:2], v[:2]) == O.OK
    before = o.state()
    assert o.tbe(np.zeros(3, np.int32), np.arange(3, dtype=np.int32),
                 np.array([0, 0, 0], np.uint8)) == O.ERR_INVALID
    assert o.tbe(seq, np.arange(2, dtype=np.int32), np.array([2, 2], np.uint8)) == O.ERR_INVALID
    after = o.state()
    assert np.array_equal(before["nseg"], after["nseg"])

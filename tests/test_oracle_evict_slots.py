"""Pins of the oracle's explicit-victim eviction (or_evict_slots):

- a small history worked by hand: the masks, free-stack pushes and FIFO
  tombstones the victims leave, and how a later budget eviction steps over
  those tombstones;
- against the budget rule: naming exactly the victims the budget rule takes
  (oldest first, T, then E, then R) gives its live set, masks, slot positions,
  live lists and free stacks, with tombstones where the budget rule moved the
  FIFO head;
- against TBE: naming, class by class, the victims TBE pushed (in its push
  order) after each append reproduces TBE's whole cache state, FIFO
  tombstones included;
- repeats and already-evicted victims are skipped, and invalid calls change
  nothing.
"""
import numpy as np

from oracle import oracle as O

import harness as Hn

R, E, T = 0, 1, 2
GEO = dict(num_q_heads=4, num_kv_heads=2, head_dim=64, group_size=32, bits=(8, 4, 2))


def _oracle(max_seqs=3, max_blocks=24, pool=200):
    return O.Oracle(GEO["num_q_heads"], GEO["num_kv_heads"], GEO["head_dim"], GEO["group_size"],
                    GEO["bits"], max_seqs, max_blocks, (pool, pool, pool))


def _kv(n, seed):
    rng = np.random.default_rng(seed)
    H, d = GEO["num_kv_heads"], GEO["head_dim"]
    return (rng.standard_normal((n, H, d)).astype(np.float16),
            rng.standard_normal((n, H, d)).astype(np.float16))


def _append(o, seq, pos, tag, seed):
    k, v = _kv(len(seq), seed)
    assert o.append(np.asarray(seq, np.int32), np.asarray(pos, np.int32),
                    np.asarray(tag, np.uint8), k, v) == O.OK


def _window(st, s, c):
    cap = st["fifo"].shape[2]
    h, t = int(st["fifo_head"][s, c]), int(st["fifo_tail"][s, c])
    return h, t, [int(x) for x in st["fifo"][s, c, np.arange(h, t) % cap]]


def _stack(st, s, c):
    return [int(x) for x in st["free_slots"][s, c, :int(st["free_top"][s, c])]]


def _same(a, b, keys):
    for key in keys:
        if isinstance(a[key], list):
            for x, y in zip(a[key], b[key]):
                assert np.array_equal(x, y), key
        else:
            assert np.array_equal(a[key], b[key]), key


STRUCT = ["table", "num_blocks", "live_count", "num_live", "live_list", "live_index",
          "slot_pos", "page_bump", "free_top", "free_slots", "fifo_tail"]


def test_hand_worked_victims_and_a_later_budget_evict():
    o = _oracle()
    _append(o, [0] * 5, range(5), [R] * 5, 1)   # a fresh R page: slots 0..4 in order
    st = o.state()
    assert _window(st, 0, R) == (0, 5, [0, 1, 2, 3, 4])
    top0 = int(st["free_top"][0, R])             # the page's 11 unused slots
    assert top0 == 11
    assert o.evict_slots([0, 0], [R, R], [3, 1]) == O.OK
    st = o.state()
    e = st["table"][0, 0]
    assert int(O.entry_mask(e)) == 0b10101
    page = int(O.entry_page(e))
    assert [int(st["slot_pos"][R][page, sl]) for sl in range(5)] == [0, -1, 2, -1, 4]
    assert _stack(st, 0, R)[top0:] == [3, 1]     # pushed in call order
    assert _window(st, 0, R) == (0, 5, [0, -1, 2, -1, 4])
    assert int(st["live_count"][0]) == 3
    Hn.check_slot_invariants(st, 3)
    # budget 2: the head (position 0) goes; the head then rests on the tombstone
    assert o.evict(np.array([0], np.int32), np.array([2], np.int32)) == O.OK
    st = o.state()
    assert _window(st, 0, R) == (1, 5, [-1, 2, -1, 4])
    # budget 1: the tombstone at the head is stepped over, position 2 goes
    assert o.evict(np.array([0], np.int32), np.array([1], np.int32)) == O.OK
    st = o.state()
    assert _window(st, 0, R) == (3, 5, [-1, 4])
    assert _stack(st, 0, R)[top0:] == [3, 1, 0, 2]
    assert int(st["live_count"][0]) == 1
    Hn.check_slot_invariants(st, 3)


def _random_history(o, rng, n_seqs=3, steps=6, seed0=0):
    pos = [0] * n_seqs
    for step in range(steps):
        seqs = [s for s in range(n_seqs) if rng.random() < 0.8]
        if not seqs:
            continue
        seq, ps, tags = [], [], []
        for s in seqs:
            m = int(rng.integers(1, 40))
            seq += [s] * m
            ps += list(range(pos[s], pos[s] + m))
            tags += list(rng.integers(0, 3, m))
            pos[s] += m
        _append(o, seq, ps, tags, seed0 + step)


def test_budget_victims_named_explicitly_match_the_budget_rule():
    for trial in range(4):
        rng_a, rng_b = np.random.default_rng(trial), np.random.default_rng(trial)
        a, b = _oracle(), _oracle()
        _random_history(a, rng_a, seed0=10 * trial)
        _random_history(b, rng_b, seed0=10 * trial)
        st = b.state()
        budgets = np.array([int(st["live_count"][s]) // (2 + trial) for s in range(3)], np.int32)
        assert a.evict(np.arange(3, dtype=np.int32), budgets) == O.OK
        # the budget rule's victims, oldest first, T then E then R (no tombstones yet)
        seq, cls, idx = [], [], []
        for s in range(3):
            nv = int(st["live_count"][s]) - int(budgets[s])
            for c in (T, E, R):
                h, t, _ = _window(st, s, c)
                take = min(nv, t - h)
                seq += [s] * take
                cls += [c] * take
                idx += list(range(h, h + take))
                nv -= take
        assert len(idx) > 0
        assert b.evict_slots(seq, cls, idx) == O.OK
        sa, sb = a.state(), b.state()
        _same(sa, sb, STRUCT)
        for s in range(3):
            for c in range(3):
                ha, ta, wa = _window(sa, s, c)
                hb, tb, wb = _window(sb, s, c)
                assert ta == tb and hb <= ha
                assert wb == [-1] * (ha - hb) + wa  # tombstones where the head moved
        Hn.check_slot_invariants(sb, 3)


def test_tbe_victims_named_explicitly_reproduce_tbe():
    named = 0
    for trial in range(3):
        rng = np.random.default_rng(100 + trial)
        a, b = _oracle(), _oracle()
        pos = [0, 0, 0]
        for step in range(40):
            seq, ps, tags = [], [], []
            for s in range(3):
                m = int(rng.integers(0, 12))
                # tags in runs, so that segments and T events form
                run_tag = int(rng.integers(0, 3))
                for _ in range(m):
                    if rng.random() < 0.25:
                        run_tag = int(rng.integers(0, 3))
                    seq.append(s)
                    ps.append(pos[s])
                    tags.append(run_tag)
                    pos[s] += 1
            if not seq:
                continue
            _append(a, seq, ps, tags, 1000 * trial + step)
            _append(b, seq, ps, tags, 1000 * trial + step)
            before = a.state()
            assert a.tbe(np.array(seq, np.int32), np.array(ps, np.int32),
                         np.array(tags, np.uint8), t_min=2, schedule=(8, 4, 2)) == O.OK
            after = a.state()
            # TBE's victims: the new free-stack entries, per class in push order,
            # each named by its FIFO counter in the state before TBE
            vs, vc, vi = [], [], []
            for s in range(3):
                for c in range(3):
                    pushed = _stack(after, s, c)[int(before["free_top"][s, c]):]
                    h, t, win = _window(before, s, c)
                    where = {x: h + j for j, x in enumerate(win) if x >= 0}
                    for ts in pushed:
                        vs.append(s)
                        vc.append(c)
                        vi.append(where[ts])
            assert b.evict_slots(vs, vc, vi) == O.OK
            named += len(vi)
            sb = b.state()
            _same(after, sb, STRUCT + ["fifo", "fifo_head"])
            Hn.check_slot_invariants(sb, 3)
    assert named > 100


def test_repeats_and_tombstones_are_skipped():
    a, b = _oracle(), _oracle()
    for o in (a, b):
        _append(o, [0] * 20 + [1] * 20, list(range(20)) * 2, [R, E, T, R] * 10, 7)
    assert a.evict_slots([0, 0, 1], [R, E, T], [2, 1, 3]) == O.OK
    assert b.evict_slots([0, 0, 0, 0, 1, 1], [R, E, R, E, T, T], [2, 1, 2, 1, 3, 3]) == O.OK
    sa = a.state()
    _same(sa, b.state(), STRUCT + ["fifo", "fifo_head"])
    # naming them again changes nothing
    assert b.evict_slots([0, 1], [R, T], [2, 3]) == O.OK
    _same(sa, b.state(), STRUCT + ["fifo", "fifo_head"])


def test_invalid_calls_change_nothing():
    o = _oracle()
    _append(o, [0] * 10 + [1] * 10, list(range(10)) * 2, [R] * 20, 3)
    st0 = o.state()
    bad = [
        ([0], [R], [10]),            # at the tail
        ([0], [R], [-1]),            # below the head
        ([0], [E], [0]),             # an empty class window
        ([0], [3], [0]),             # no such class
        ([3], [R], [0]),             # sequence out of range
        ([0, 1, 0], [R, R, R], [0, 0, 1]),   # sequence 0 in two runs
    ]
    for seq, cls, idx in bad:
        assert o.evict_slots(seq, cls, idx) == O.ERR_INVALID, (seq, cls, idx)
        _same(st0, o.state(), STRUCT + ["fifo", "fifo_head"])
    assert o.evict_slots([], [], []) == O.OK
    _same(st0, o.state(), STRUCT + ["fifo", "fifo_head"])

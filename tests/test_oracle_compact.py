"""Pins of the oracle's gather compaction (the step CT avoids): a hand-worked
example, hole-free pages, FIFO order and positions carried over, and
placement invariance -- decode over the compacted copy equals decode over the
original bit for bit -- on histories with budget evictions and TBE
tombstones."""
import numpy as np
import pytest

from oracle import oracle as O

import harness as Hn


def _kv(n, H, d, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, H, d)).astype(np.float16),
            rng.standard_normal((n, H, d)).astype(np.float16))


def test_hand_worked_compaction():
    """One sequence: tags R R E R T E E R R T at positions 0..9, evicted to 6
    (T first, then E, oldest first: victims 4, 9, 2, 5), then compacted.
    Worked by hand: R tokens 0, 1, 3, 7, 8 fill slots 0-4 of dst R page 0
    (entry 0), E token 6 slot 0 of dst E page 0 (entry 1); the free stacks
    hold the rest of each last page, lowest slot on top."""
    o = O.Oracle(2, 1, 64, 32, (8, 4, 2), 1, 8, (4, 4, 4))
    d = O.Oracle(2, 1, 64, 32, (8, 4, 2), 1, 8, (4, 4, 4))
    tags = np.array([0, 0, 1, 0, 2, 1, 1, 0, 0, 2], np.uint8)
    k, v = _kv(10, 1, 64, 3)
    assert o.append(np.zeros(10, np.int32), np.arange(10, dtype=np.int32), tags, k, v) == O.OK
    assert o.evict(np.zeros(1, np.int32), np.array([6], np.int32)) == O.OK
    assert o.compact_into(d, np.zeros(1, np.int32)) == O.OK
    st = d.state()
    assert st["page_bump"].tolist() == [1, 1, 0]
    assert int(st["num_blocks"][0]) == 2 and int(st["num_live"][0]) == 2
    assert int(st["live_count"][0]) == 6
    t = st["table"][0, :2]
    assert O.entry_class(t).tolist() == [0, 1] and O.entry_page(t).tolist() == [0, 0]
    assert O.entry_mask(t).tolist() == [0b11111, 0b1]
    assert st["slot_pos"][0][0, :5].tolist() == [0, 1, 3, 7, 8]
    assert st["slot_pos"][0][0, 5:].tolist() == [-1] * 11
    assert st["slot_pos"][1][0, :2].tolist() == [6, -1]
    assert st["fifo"][0, 0, :5].tolist() == [0, 1, 2, 3, 4] and st["fifo"][0, 1, :1].tolist() == [16]
    assert st["fifo_tail"][0].tolist() == [5, 1, 0] and st["fifo_head"][0].tolist() == [0, 0, 0]
    assert st["free_top"][0].tolist() == [11, 15, 0]
    assert st["free_slots"][0, 0, :11].tolist() == list(range(15, 4, -1))
    assert st["free_slots"][0, 1, :15].tolist() == list(range(31, 16, -1))
    # codes moved, not requantised: E token 6 sat in slot 2 of the source E
    # page (E tokens 2, 5, 6 took slots 0, 1, 2); it is now slot 0 of dst's
    so = o.state()
    src_page = int(O.entry_page(so["table"][0, 1]))
    assert int(O.entry_class(so["table"][0, 1])) == 1
    assert np.array_equal(d.codes(1)[0, :, :, 0], o.codes(1)[src_page, :, :, 2])
    assert np.array_equal(d.params(1)[0, :, :, 0], o.params(1)[src_page, :, :, 2])


@pytest.mark.parametrize("seed", range(5))
def test_compaction_is_placement_invariant(seed):
    rng = np.random.default_rng(seed)
    ns, L, H, dd = 4, 500, 2, 64
    bits = [(8, 4, 2), (16, 4, 2), (2, 8, 16)][seed % 3]
    nb = L // 16 * 3 + 8
    pool = (ns * L // 16 + 8,) * 3
    o = O.Oracle(8, H, dd, 32, bits, ns, nb, pool)
    d = O.Oracle(8, H, dd, 32, bits, ns, nb, pool)
    for p0 in range(0, L, 100):
        seq = np.repeat(np.arange(ns, dtype=np.int32), 100)
        pos = np.tile(np.arange(p0, p0 + 100, dtype=np.int32), ns)
        tag = np.repeat(rng.integers(0, 3, ns * 100 // 5), 5).astype(np.uint8)
        k, v = _kv(len(seq), H, dd, 10 + p0)
        assert o.append(seq, pos, tag, k, v) == O.OK
        assert o.tbe(seq, pos, tag, t_min=3, schedule=[20, 10, 5]) == O.OK
        b = rng.integers(50, 300, ns).astype(np.int32)
        assert o.evict(np.arange(ns, dtype=np.int32), b) == O.OK
    order = rng.permutation(ns).astype(np.int32)
    assert o.compact_into(d, order) == O.OK
    so, sd = o.state(), d.state()
    Hn.check_slot_invariants(sd, ns)
    for s in range(ns):
        # hole-free: every page but the last of each class is full
        t = sd["table"][s, :int(sd["num_blocks"][s])]
        for c in range(3):
            m = O.entry_mask(t[O.entry_class(t) == c])
            assert np.all(m[:-1] == 0xFFFF)
        # the FIFO windows carry the same positions in the same order
        for c in range(3):
            def positions(st, who):
                cap = st["fifo"].shape[2]
                h, tl = int(st["fifo_head"][who, c]), int(st["fifo_tail"][who, c])
                out = []
                for x in st["fifo"][who, c, np.arange(h, tl) % cap]:
                    if x < 0:
                        continue
                    page = int(O.entry_page(st["table"][who, int(x) // 16]))
                    out.append(int(st["slot_pos"][c][page, int(x) % 16]))
                return out
            assert positions(so, s) == positions(sd, s)
        assert int(sd["live_count"][s]) == int(so["live_count"][s])
    q = np.random.default_rng(99).standard_normal((ns, 8, dd)).astype(np.float16)
    ids = np.arange(ns, dtype=np.int32)
    r1, m1 = o.decode(ids, q, topk=6, threads=4)
    r2, m2 = d.decode(ids, q, topk=6, threads=4)
    assert np.array_equal(r1, r2) and np.array_equal(m1, m2)


def test_compaction_rejects_bad_calls():
    o = O.Oracle(2, 1, 64, 32, (8, 4, 2), 2, 8, (4, 4, 4))
    d = O.Oracle(2, 1, 64, 32, (8, 4, 2), 2, 8, (4, 4, 4))
    small = O.Oracle(2, 1, 64, 32, (8, 4, 2), 2, 8, (1, 1, 1))
    k, v = _kv(40, 1, 64, 1)
    seq = np.repeat(np.arange(2, dtype=np.int32), 20)
    pos = np.tile(np.arange(20, dtype=np.int32), 2)
    assert o.append(seq, pos, np.zeros(40, np.uint8), k, v) == O.OK
    assert o.compact_into(d, np.array([0, 0], np.int32)) == O.ERR_INVALID
    assert o.compact_into(d, np.array([0, 2], np.int32)) == O.ERR_INVALID
    assert o.compact_into(small, np.array([0, 1], np.int32)) == O.ERR_OUT_OF_PAGES
    assert o.compact_into(d, np.array([1], np.int32)) == O.OK
    assert o.compact_into(d, np.array([1], np.int32)) == O.ERR_INVALID      # dst not empty for 1

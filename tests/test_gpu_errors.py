"""Device-detected errors of append and evict, on both launch paths (calls of
at most 512 tokens or sequences take a one-launch path; larger calls the
single-CTA bookkeeping kernels): the status code matches the oracle's for the
same call, the call changes nothing (all-or-nothing), a set status makes
later appends and evicts do nothing, and clearing it makes them work again.
Also: one-launch calls whose runs hold many tokens match the oracle bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from mixed_precision_paged_thinkv_b200 import workloads as W
from mixed_precision_paged_thinkv_b200.binding import ThinKVCache

import harness as Hn

pytestmark = pytest.mark.gpu

HQ, HKV, D, G = 4, 2, 64, 32


def _pair(max_seqs, max_blocks, pool, bits=(8, 4, 2)):
    g = ThinKVCache(HQ, HKV, D, G, bits, max_seqs, max_blocks, pool)
    o = O.Oracle(HQ, HKV, D, G, bits, max_seqs, max_blocks, pool)
    return g, o


def _kv(n, seed):
    gen = torch.Generator().manual_seed(seed)
    k = torch.randn(n, HKV, D, generator=gen).half()
    v = torch.randn(n, HKV, D, generator=gen).half()
    return k, v


def _append_both(g, o, seq, pos, tag, seed=0):
    seq = np.asarray(seq, dtype=np.int32)
    pos = np.asarray(pos, dtype=np.int32)
    tag = np.asarray(tag, dtype=np.uint8)
    k, v = _kv(len(seq), seed)
    dev = g.device
    g.append(torch.as_tensor(seq, device=dev), torch.as_tensor(pos, device=dev),
             torch.as_tensor(tag, device=dev), k.to(dev), v.to(dev))
    return o.append(seq, pos, tag, k, v)


def _evict_both(g, o, seq, budget):
    seq = np.asarray(seq, dtype=np.int32)
    budget = np.asarray(budget, dtype=np.int32)
    dev = g.device
    g.evict(torch.as_tensor(seq, device=dev), torch.as_tensor(budget, device=dev))
    return o.evict(seq, budget)


def _same(g, o, ns):
    torch.cuda.synchronize()
    Hn.compare_state(g.snapshot(), o.state(), ns)


def _history(g, o, ns, per_seq, seed=1):
    """A valid history: per_seq tokens for each of ns sequences, one call."""
    rng = np.random.default_rng(seed)
    seq = np.repeat(np.arange(ns), per_seq)
    pos = np.tile(np.arange(per_seq), ns)
    tag = rng.integers(0, 3, size=seq.size)
    assert _append_both(g, o, seq, pos, tag, seed) == O.OK
    assert g.status() == 0
    assert _evict_both(g, o, np.arange(ns), np.full(ns, per_seq // 2)) == O.OK
    assert g.status() == 0
    _same(g, o, ns)


# (n tokens per call) small path: 6 sequences x 20; general path: 6 x 200
@pytest.mark.parametrize("per_seq", [20, 200])
def test_bad_append_data_is_rejected_and_changes_nothing(per_seq):
    ns = 6
    g, o = _pair(ns, 64, (200, 200, 200))
    _history(g, o, ns, per_seq)
    before = g.snapshot()
    L = per_seq
    cases = {
        "sequence out of range": ([0, 1, ns], [L, L, L], [0, 1, 2]),
        "tag 3": ([0, 1, 2], [L, L, L], [0, 3, 1]),
        "negative position": ([0, 1, 2], [L, -1, L], [0, 0, 0]),
        "positions not ascending": ([0, 0, 1], [L + 1, L + 1, L], [0, 1, 2]),
        "sequence in two runs": ([0, 1, 0], [L, L, L + 1], [0, 1, 2]),
    }
    for what, (seq, pos, tag) in cases.items():
        # pad to the path under test with valid tokens of other sequences
        if per_seq > 100:
            extra = np.arange(3, ns)
            seq = list(seq) + list(np.repeat(extra, 200))
            pos = list(pos) + list(np.tile(np.arange(L, L + 200), len(extra)))
            tag = list(tag) + [0] * (200 * len(extra))
        st = _append_both(g, o, seq, pos, tag, seed=7)
        torch.cuda.synchronize()
        assert st == O.ERR_INVALID, what
        assert g.status() == O.ERR_INVALID, what
        after = g.snapshot()
        for key in before:
            if key == "slot_pos":
                assert all(np.array_equal(a, b) for a, b in zip(before[key], after[key])), what
            else:
                assert np.array_equal(before[key], after[key]), (what, key)
        g.clear_status()
    _same(g, o, ns)


@pytest.mark.parametrize("per_seq", [20, 200])
def test_out_of_pages_and_out_of_blocks(per_seq):
    ns = 4
    # pools sized for the history plus almost nothing
    g, o = _pair(ns, 64, (30, 30, 30) if per_seq == 20 else (60, 60, 60))
    _history(g, o, ns, per_seq)
    before = g.snapshot()
    n_new = 512 if per_seq == 20 else 1200
    seq = np.repeat(np.arange(ns), n_new // ns)
    pos = np.tile(np.arange(per_seq, per_seq + n_new // ns), ns)
    tag = np.zeros(seq.size, dtype=np.uint8)             # all R: one pool runs dry
    st = _append_both(g, o, seq, pos, tag, seed=9)
    torch.cuda.synchronize()
    assert st == O.ERR_OUT_OF_PAGES
    assert g.status() == O.ERR_OUT_OF_PAGES
    after = g.snapshot()
    assert np.array_equal(before["table"], after["table"])
    assert np.array_equal(before["page_bump"], after["page_bump"])
    g.clear_status()
    _same(g, o, ns)

    g2, o2 = _pair(ns, 8, (500, 500, 500))               # 8 table entries per sequence
    rng = np.random.default_rng(3)
    seq = np.repeat(np.arange(ns), 40)
    pos = np.tile(np.arange(40), ns)
    tag = rng.integers(0, 3, size=seq.size)
    assert _append_both(g2, o2, seq, pos, tag, seed=2) == O.OK
    big = 120 if per_seq == 20 else 200
    seq = np.repeat(np.arange(ns), big)
    pos = np.tile(np.arange(40, 40 + big), ns)
    st = _append_both(g2, o2, seq, pos, np.zeros(seq.size, dtype=np.uint8), seed=4)
    torch.cuda.synchronize()
    assert st == O.ERR_OUT_OF_BLOCKS
    assert g2.status() == O.ERR_OUT_OF_BLOCKS
    g2.clear_status()
    _same(g2, o2, ns)


@pytest.mark.parametrize("ns", [6, 700])
def test_bad_evict_data_is_rejected_and_changes_nothing(ns):
    g, o = _pair(ns, 16, (ns * 4, ns * 4, ns * 4))
    _history(g, o, ns, 20)
    before = g.snapshot()
    base_seq = list(range(ns))
    for what, (seq, bud) in {
        "duplicate sequence": (base_seq[:-1] + [0], [3] * ns),
        "negative budget": (base_seq, [3] * (ns - 1) + [-1]),
        "sequence out of range": (base_seq[:-1] + [ns], [3] * ns),
    }.items():
        st = _evict_both(g, o, seq, bud)
        torch.cuda.synchronize()
        assert st == O.ERR_INVALID, what
        assert g.status() == O.ERR_INVALID, what
        after = g.snapshot()
        assert np.array_equal(before["table"], after["table"]), what
        assert np.array_equal(before["live_count"], after["live_count"]), what
        g.clear_status()
    _same(g, o, ns)


def test_sticky_status_blocks_append_and_evict():
    ns = 3
    g, o = _pair(ns, 16, (40, 40, 40))
    _history(g, o, ns, 20)
    _append_both(g, o, [0, 0], [30, 29], [0, 0])       # not ascending -> INVALID (oracle too)
    torch.cuda.synchronize()
    assert g.status() == O.ERR_INVALID
    before = g.snapshot()
    k, v = _kv(3, 5)
    dev = g.device
    g.append(torch.tensor([0, 1, 2], dtype=torch.int32, device=dev),
             torch.tensor([40, 40, 40], dtype=torch.int32, device=dev),
             torch.tensor([0, 1, 2], dtype=torch.uint8, device=dev), k.to(dev), v.to(dev))
    g.evict(torch.arange(ns, dtype=torch.int32, device=dev),
            torch.zeros(ns, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    after = g.snapshot()
    assert np.array_equal(before["table"], after["table"])
    assert np.array_equal(before["live_count"], after["live_count"])
    g.clear_status()
    assert g.status() == 0
    # the oracle never saw the blocked calls; after clearing, both work again
    assert _append_both(g, o, [0, 1, 2], [40, 40, 40], [0, 1, 2], seed=11) == O.OK
    assert _evict_both(g, o, [0, 1, 2], [5, 5, 5]) == O.OK
    _same(g, o, ns)


def test_one_launch_calls_with_long_runs_match_the_oracle():
    """Calls of <= 512 tokens whose runs hold many tokens (prefill-like) go
    through the one-launch path; state and codes must match bit for bit."""
    ns = 5
    g, o = _pair(ns, 64, (120, 120, 120))
    rng = np.random.default_rng(21)
    posn = np.zeros(ns, dtype=np.int64)
    for call in range(6):
        lens = rng.integers(0, 100, size=ns)
        seqs = [s for s in range(ns) if lens[s] > 0]
        seq = np.concatenate([np.full(lens[s], s) for s in seqs])
        pos = np.concatenate([np.arange(posn[s], posn[s] + lens[s]) for s in seqs])
        tag = np.concatenate([rng.integers(0, 3, size=lens[s]) for s in seqs])
        assert seq.size <= 512
        assert _append_both(g, o, seq, pos, tag, seed=call) == O.OK
        posn += lens
        bud = (posn * rng.uniform(0.2, 0.9, size=ns)).astype(np.int32)
        assert _evict_both(g, o, np.arange(ns), bud) == O.OK
        torch.cuda.synchronize()
        assert g.status() == 0
        _same(g, o, ns)
    Hn.compare_codes(g, o, o.state(), ns)

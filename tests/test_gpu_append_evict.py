"""GPU parity of the one-call append + evict (thinkv_append_evict) against the
oracle's append followed by its evict: the whole cache state bit for bit and
every live slot's codes after each call, for calls small enough for the
one-launch path (one token per sequence, and runs of several tokens) and
larger ones, budgets from 0 to above the live count, a non-default class
order, budgets at non-first tokens ignored, and refused calls (a negative
budget, bad token data) that change nothing."""
import numpy as np
import pytest
import torch

from oracle import oracle as O

import harness as Hn

pytestmark = pytest.mark.gpu


def _pair(d, G, bits, ns, nb, pool, H=2, Hq=4):
    from mixed_precision_paged_thinkv_b200.binding import ThinKVCache
    g = ThinKVCache(Hq, H, d, G, bits, ns, nb, pool)
    o = O.Oracle(Hq, H, d, G, bits, ns, nb, pool)
    return g, o


def _dev(a, dt):
    return torch.as_tensor(np.ascontiguousarray(a)).to("cuda", dt)


def _compare(g, o, ns):
    torch.cuda.synchronize()
    assert g.status() == 0
    st = o.state()
    Hn.compare_state(g.snapshot(), st, ns)
    Hn.compare_codes(g, o, st, ns)
    return st


def _call(g, o, rng, ns, pos, H, d, per_seq, order=None, budget_frac=0.5):
    seqs = rng.permutation(ns)[: max(1, int(ns * 0.8))]
    seq, ps, tags, bud = [], [], [], []
    st = o.state()
    for s in seqs:
        m = per_seq if per_seq > 0 else int(rng.integers(1, 12))
        live_after = int(st["live_count"][s]) + m
        b = int(live_after * budget_frac) if rng.random() < 0.8 else int(rng.integers(0, live_after + 5))
        for j in range(m):
            seq.append(int(s))
            ps.append(pos[s])
            tags.append(int(rng.integers(0, 3)))
            bud.append(b if j == 0 else -1)      # only the run's first budget is read
            pos[s] += 1
    n = len(seq)
    k = torch.as_tensor(rng.standard_normal((n, H, d)).astype(np.float16))
    v = torch.as_tensor(rng.standard_normal((n, H, d)).astype(np.float16))
    seq, ps = np.array(seq, np.int32), np.array(ps, np.int32)
    tags, bud = np.array(tags, np.uint8), np.array(bud, np.int32)
    g.append_evict(_dev(seq, torch.int32), _dev(ps, torch.int32), _dev(tags, torch.uint8),
                   k.cuda(), v.cuda(), _dev(bud, torch.int32), order=order)
    assert o.append(seq, ps, tags, k.numpy(), v.numpy()) == O.OK
    starts = np.r_[True, seq[1:] != seq[:-1]]
    assert o.evict(seq[starts], bud[starts], order) == O.OK
    return n


@pytest.mark.parametrize("per_seq,order", [(1, None), (0, None), (1, (1, 2, 0))])
def test_small_calls_match_append_then_evict(per_seq, order):
    rng = np.random.default_rng(per_seq * 10 + (order is not None))
    ns, H, d = 40, 2, 64
    g, o = _pair(d, 32, (8, 4, 2), ns, 64, (900, 900, 900), H=H)
    pos = [0] * ns
    for step in range(12):
        n = _call(g, o, rng, ns, pos, H, d, per_seq, order=order, budget_frac=[0.9, 0.5, 0.2][step % 3])
        assert n <= 512
        _compare(g, o, ns)
    st = o.state()
    Hn.check_slot_invariants(st, ns)


def test_large_calls_match_append_then_evict():
    rng = np.random.default_rng(7)
    ns, H, d = 24, 2, 128
    g, o = _pair(d, 64, (4, 2, 8), ns, 96, (1200, 1200, 1200), H=H, Hq=8)
    pos = [0] * ns
    for step in range(4):
        n = _call(g, o, rng, ns, pos, H, d, per_seq=40, budget_frac=[0.7, 0.4][step % 2])
        assert n > 512                           # the two-kernel append, then the evict kernel
        _compare(g, o, ns)


def test_refused_calls_change_nothing():
    rng = np.random.default_rng(3)
    ns, H, d = 8, 2, 64
    g, o = _pair(d, 32, (8, 4, 2), ns, 32, (300, 300, 300), H=H)
    pos = [0] * ns
    _call(g, o, rng, ns, pos, H, d, per_seq=5)
    st = _compare(g, o, ns)
    k = torch.zeros(2, H, d, dtype=torch.float16, device="cuda")
    for seq, p, bud in [([0, 1], [pos[0], pos[1]], [3, -1]),         # a run's budget negative
                        ([0, 0], [pos[0], pos[0]], [3, 3]),          # positions not increasing
                        ([0, ns], [pos[0], 0], [3, 3])]:             # sequence out of range
        g.append_evict(_dev(seq, torch.int32), _dev(p, torch.int32), _dev([0, 0], torch.uint8),
                       k, k, _dev(bud, torch.int32))
        torch.cuda.synchronize()
        assert g.status() == O.ERR_INVALID
        g.clear_status()
        Hn.compare_state(g.snapshot(), st, ns)

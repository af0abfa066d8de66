"""GPU parity of explicit victims (thinkv_evict_slots) against the oracle: the
whole cache state bit for bit after every call (tables, free stacks in push
order, FIFO windows with their tombstones, live lists, slot positions), with
victims named in batches longer than a warp, repeats inside and across
batches, victims already evicted, budget evictions stepping over the
tombstones afterwards, refused calls, and decode on the resulting states
within 2e-3."""
import numpy as np
import pytest
import torch

from oracle import oracle as O

import harness as Hn

pytestmark = pytest.mark.gpu


def _pair(Hq, Hkv, d, G, bits, ns, nb, pool):
    from mixed_precision_paged_thinkv_b200.binding import ThinKVCache
    g = ThinKVCache(Hq, Hkv, d, G, bits, ns, nb, pool)
    o = O.Oracle(Hq, Hkv, d, G, bits, ns, nb, pool)
    return g, o


def _dev(a, dt):
    return torch.as_tensor(np.ascontiguousarray(a)).to("cuda", dt)


def _compare(g, o, ns):
    torch.cuda.synchronize()
    assert g.status() == 0
    gs, os_ = g.snapshot(), o.state()
    Hn.compare_state(gs, os_, ns)
    Hn.compare_codes(g, o, os_, ns)
    return os_


def _append(g, o, rng, ns, pos, H, d):
    seq, ps, tags = [], [], []
    for s in range(ns):
        m = int(rng.integers(0, 60))
        run = int(rng.integers(0, 3))
        for _ in range(m):
            if rng.random() < 0.2:
                run = int(rng.integers(0, 3))
            seq.append(s)
            ps.append(pos[s])
            tags.append(run)
            pos[s] += 1
    if not seq:
        return
    n = len(seq)
    k = torch.as_tensor(rng.standard_normal((n, H, d)).astype(np.float16))
    v = torch.as_tensor(rng.standard_normal((n, H, d)).astype(np.float16))
    seq, ps, tags = np.array(seq, np.int32), np.array(ps, np.int32), np.array(tags, np.uint8)
    g.append(_dev(seq, torch.int32), _dev(ps, torch.int32), _dev(tags, torch.uint8), k.cuda(), v.cuda())
    assert o.append(seq, ps, tags, k.numpy(), v.numpy()) == O.OK


def _victims(st, rng, ns, frac):
    """Random victims per sequence (a run each, sequences in random order):
    counters anywhere in the FIFO windows, tombstones included, some named twice."""
    order = rng.permutation(ns)
    seq, cls, idx = [], [], []
    for s in order:
        cand = []
        for c in range(3):
            h, t = int(st["fifo_head"][s, c]), int(st["fifo_tail"][s, c])
            cand += [(c, k) for k in range(h, t)]
        if not cand:
            continue
        m = int(len(cand) * frac)
        pick = [cand[j] for j in rng.choice(len(cand), size=m, replace=False)]
        pick += [pick[j] for j in rng.choice(len(pick), size=len(pick) // 8)] if pick else []
        rng.shuffle(pick)
        for c, k in pick:
            seq.append(int(s))
            cls.append(c)
            idx.append(k)
    return np.array(seq, np.int32), np.array(cls, np.uint8), np.array(idx, np.int32)


@pytest.mark.parametrize("d,G,bits", [(64, 32, (8, 4, 2)), (128, 64, (4, 2, 8))])
def test_explicit_victims_match_the_oracle(d, G, bits):
    rng = np.random.default_rng(d + bits[0])
    ns, H = 5, 2
    g, o = _pair(8, H, d, G, bits, ns, 48, (400, 400, 400))
    pos = [0] * ns
    total = 0
    for step in range(8):
        _append(g, o, rng, ns, pos, H, d)
        st = _compare(g, o, ns)
        seq, cls, idx = _victims(st, rng, ns, frac=[0.1, 0.4, 0.7][step % 3])
        total += len(idx)
        g.evict_slots(_dev(seq, torch.int32), _dev(cls, torch.uint8), _dev(idx, torch.int32))
        assert o.evict_slots(seq, cls, idx) == O.OK
        st = _compare(g, o, ns)
        Hn.check_slot_invariants(st, ns)
        if step % 2:
            # the budget rule steps over the tombstones the victims left
            b = np.array([int(st["live_count"][s]) * 3 // 4 for s in range(ns)], np.int32)
            g.evict(_dev(np.arange(ns), torch.int32), _dev(b, torch.int32))
            assert o.evict(np.arange(ns, dtype=np.int32), b) == O.OK
            _compare(g, o, ns)
    assert total > 300
    # decode over the state with its holes and tombstones
    q = torch.as_tensor(rng.standard_normal((ns, 8, d)).astype(np.float16))
    out, _ = g.decode(_dev(np.arange(ns), torch.int32), q.cuda())
    ref, _ = o.decode(np.arange(ns, dtype=np.int32), q.numpy())
    assert Hn.attn_error(out.cpu().numpy(), ref) <= Hn.TOL


def test_refused_calls_change_nothing():
    rng = np.random.default_rng(5)
    ns, H, d = 3, 2, 64
    g, o = _pair(4, H, d, 32, (8, 4, 2), ns, 24, (200, 200, 200))
    pos = [0] * ns
    _append(g, o, rng, ns, pos, H, d)
    st = _compare(g, o, ns)
    s = int(np.argmax(st["live_count"]))
    c = int(np.argmax(st["fifo_tail"][s] - st["fifo_head"][s]))
    t = int(st["fifo_tail"][s, c])
    bad = [([s], [c], [t]), ([s], [3], [0]), ([ns + 7], [c], [0]),
           ([s, (s + 1) % ns, s], [c, c, c], [t - 1, 0, t - 2])]
    for seq, cls, idx in bad:
        seq, cls, idx = np.array(seq, np.int32), np.array(cls, np.uint8), np.array(idx, np.int32)
        assert o.evict_slots(seq, cls, idx) == O.ERR_INVALID
        g.evict_slots(_dev(seq, torch.int32), _dev(cls, torch.uint8), _dev(idx, torch.int32))
        torch.cuda.synchronize()
        assert g.status() == O.ERR_INVALID
        g.clear_status()
        Hn.compare_state(g.snapshot(), o.state(), ns)

"""GPU parity of TBE (thinkv_evict_tbe) and of the tombstone-aware budget
evict against the oracle: the whole cache state bit for bit after every
operation (tables, free stacks, FIFO windows with their tombstones, live
lists, slot positions, segment records), then decode on the states TBE
leaves, within 2e-3."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from mixed_precision_paged_thinkv_b200 import workloads as W

import harness as Hn

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
CLS = {"R": 0, "E": 1, "T": 2}


def _pair(Hq, Hkv, d, G, bits, ns, nb, pool):
    from mixed_precision_paged_thinkv_b200.binding import ThinKVCache
    g = ThinKVCache(Hq, Hkv, d, G, bits, ns, nb, pool, tbe=True)
    o = O.Oracle(Hq, Hkv, d, G, bits, ns, nb, pool)
    return g, o


def _compare(g, o, ns):
    torch.cuda.synchronize()
    assert g.status() == 0
    gs, os_ = g.snapshot(), o.state()
    Hn.compare_state(gs, os_, ns)
    assert np.array_equal(gs["nseg"], os_["nseg"])
    for s in range(ns):
        k = int(os_["nseg"][s])
        assert np.array_equal(gs["seg"][s, :k], os_["seg"][s, :k]), f"segments of seq {s}"
    return gs


def _dev(a, dt):
    return torch.as_tensor(np.ascontiguousarray(a)).to("cuda", dt)


def _call(g, o, seq, pos, tag, k, v, t_min, schedule):
    g.append(_dev(seq, torch.int32), _dev(pos, torch.int32), _dev(tag, torch.uint8),
             k.cuda(), v.cuda())
    g.evict_tbe(_dev(seq, torch.int32), _dev(pos, torch.int32), _dev(tag, torch.uint8),
                t_min=t_min, schedule=schedule)
    assert o.append(seq, pos, tag, k, v) == O.OK
    assert o.tbe(seq, pos, tag, t_min=t_min, schedule=schedule) == O.OK


@pytest.mark.parametrize("per_token", [False, True])
def test_hand_worked_history_on_gpu(per_token):
    gold = json.load(open(os.path.join(HERE, "golden", "tbe_example.json")))
    geo = gold["geometry"]
    g, o = _pair(geo["num_q_heads"], geo["num_kv_heads"], geo["head_dim"], geo["group_size"],
                 geo["bits"], geo["max_seqs"], geo["max_blocks_per_seq"], geo["pool_pages"])
    tags = np.array([CLS[t] for t in gold["tags"]], dtype=np.uint8)
    rng = np.random.default_rng(0)
    kk = torch.as_tensor(rng.standard_normal((len(tags), 1, 64)).astype(np.float16))
    vv = torch.as_tensor(rng.standard_normal((len(tags), 1, 64)).astype(np.float16))
    for step in gold["steps"]:
        if step["op"] == "append+tbe":
            a, b = step["positions"]
            for (p0, p1) in ([(p, p + 1) for p in range(a, b)] if per_token else [(a, b)]):
                seq = np.zeros(p1 - p0, np.int32)
                pos = np.arange(p0, p1, dtype=np.int32)
                _call(g, o, seq, pos, tags[p0:p1], kk[p0:p1].contiguous(), vv[p0:p1].contiguous(),
                      gold["t_min"], gold["schedule"])
        else:
            b = np.array([step["budget"]], np.int32)
            g.evict(_dev(np.zeros(1, np.int32), torch.int32), _dev(b, torch.int32))
            assert o.evict(np.zeros(1, np.int32), b) == O.OK
        gs = _compare(g, o, 1)
        assert int(gs["live_count"][0]) == step["live_count"]


@pytest.mark.parametrize("seed", range(6))
def test_random_histories_with_budget_evictions(seed):
    rng = np.random.default_rng(200 + seed)
    ns, L, H, d, G = 4, 900, 2, 64, 32
    bits = [(8, 4, 2), (16, 8, 4), (4, 2, 8)][seed % 3]
    schedule = [int(x) for x in sorted(rng.integers(1, 40, 3), reverse=True)]
    t_min = int(rng.integers(0, 10))
    tags = {}
    for s in range(ns):
        t = []
        while len(t) < L:
            t += [int(rng.choice(3, p=[0.35, 0.4, 0.25]))] * int(rng.integers(1, 30))
        tags[s] = np.array(t[:L], np.uint8)
    g, o = _pair(8, H, d, G, bits, ns, L // 16 * 3 + 8, (ns * L // 16 + 8,) * 3)
    done = [0] * ns
    step = 0
    while min(done) < L:
        seqs, poss, tg = [], [], []
        big = step < 3
        for s in rng.permutation(ns).tolist():
            if done[s] >= L:
                continue
            cnt = int(min(L - done[s], rng.integers(100, 300) if big else rng.integers(1, 6)))
            seqs += [s] * cnt
            poss += list(range(done[s], done[s] + cnt))
            tg += tags[s][done[s]:done[s] + cnt].tolist()
            done[s] += cnt
        seqs, poss, tg = np.array(seqs, np.int32), np.array(poss, np.int32), np.array(tg, np.uint8)
        kv = rng.standard_normal((2, len(seqs), H, d)).astype(np.float16)
        _call(g, o, seqs, poss, tg, torch.as_tensor(kv[0]), torch.as_tensor(kv[1]), t_min, schedule)
        if rng.random() < 0.35:
            st = o.state()
            sel = np.sort(rng.choice(ns, size=int(rng.integers(1, ns + 1)), replace=False)).astype(np.int32)
            b = np.array([int(rng.integers(0, int(st["live_count"][s]) + 1)) for s in sel], np.int32)
            order = [int(x) for x in rng.permutation(3)]
            g.evict(_dev(sel, torch.int32), _dev(b, torch.int32), order=order)
            assert o.evict(sel, b, order=order) == O.OK
        if step % 7 == 0 or min(done) >= L:
            _compare(g, o, ns)
        step += 1
    gs = _compare(g, o, ns)
    Hn.check_slot_invariants(gs, ns)
    q = torch.as_tensor(rng.standard_normal((ns, 8, d)).astype(np.float16))
    out, mass = g.decode(torch.arange(ns, dtype=torch.int32, device="cuda"), q.cuda(), topk=8)
    ref, rmass = o.decode(np.arange(ns, dtype=np.int32), q, topk=8, threads=8)
    err = Hn.attn_error(out.cpu().numpy(), ref)
    merr = float(np.abs(mass.cpu().numpy().astype(np.float64) - rmass).max())
    print(f"TBE seed {seed}: attention error {err:.3e}, top-k mass error {merr:.3e}")
    assert err <= Hn.TOL and merr <= Hn.MASS_TOL


def test_tbe_on_a_reduced_llama_shaped_layer():
    """The R1-Distill-Llama-8B layer shape, 4 sequences of 6000 generated
    tokens, default schedule (64, 32, 16) and a safety net of 16 T tokens:
    prefill calls of 2048 positions with TBE after each, then 40 decode steps
    of (append one token, TBE, decode)."""
    w = W.scaled(W.WORKLOADS["r1-llama-8b"], batch=4, lengths=("fixed", 6000))
    sched = W.Schedule(w, extra=41)
    L = 6000 + 41
    g, o = _pair(w.num_q_heads, w.num_kv_heads, w.head_dim, w.group_size, w.bits, 4,
                 L // 16 * 2 + 8, (4 * L // 16 + 8,) * 3)
    for p0 in range(0, 6000, 2048):
        runs = [(s, p0, min(2048, 6000 - p0)) for s in range(4)]
        call = W.make_append_call(runs, sched.tags)
        k, v = W.call_kv(w, call)
        _call(g, o, call.seqs, call.pos, call.tags, k, v, 16, None)
    _compare(g, o, 4)
    gen = np.full(4, 6000)
    for step in range(40):
        call = sched.one_token_call(gen)
        k, v = W.call_kv(w, call)
        _call(g, o, call.seqs, call.pos, call.tags, k, v, 16, None)
        gen += 1
        q = W.q_values(w, step)[:4].contiguous()
        out, _ = g.decode(torch.arange(4, dtype=torch.int32, device="cuda"), q.cuda())
        if step % 10 == 9:
            _compare(g, o, 4)
            ref, _ = o.decode(np.arange(4, dtype=np.int32), q, threads=8)
            err = Hn.attn_error(out.cpu().numpy(), ref)
            print(f"llama-shaped TBE step {step}: attention error {err:.3e}, "
                  f"live {o.state()['live_count'].tolist()}")
            assert err <= Hn.TOL

"""GPU parity: libthinkv (CUDA, sm_100a, through the C ABI) against the oracle.

Bit-exact: block tables, free stacks, FIFOs, live lists, slot positions, page
counters, and the codes/params of every live slot.  Decode outputs: within
2e-3 row-normalised max error of the oracle's fp64 attention on the same
dequantised values; top-k mass within 2e-3 absolute.
"""
import numpy as np
import pytest
import torch

from mixed_precision_paged_thinkv_b200 import workloads as W

import harness as Hn

pytestmark = pytest.mark.gpu


def _pair(w, extra=0, bits=None):
    from mixed_precision_paged_thinkv_b200.runner import WorkloadRun
    g = WorkloadRun(w, extra=extra, bits=bits)
    o = Hn.OracleRun(w, g.geom, extra=extra, bits=bits)
    return g, o


def _check_all(g, o, step=0, topk=None, codes=True, max_pages=None):
    torch.cuda.synchronize()
    assert g.cache.status() == 0
    gs = g.cache.snapshot()
    os_ = o.o.state()
    Hn.compare_state(gs, os_, g.w.batch)
    if codes:
        Hn.compare_codes(g.cache, o.o, os_, g.w.batch, max_pages=max_pages)
    out, mass = g.decode(step, topk=topk)
    ref, rmass = o.decode(step, topk=topk)
    err = Hn.attn_error(out.cpu().numpy(), ref)
    print(f"{g.w.name} step {step}: attention error {err:.3e}")
    assert err <= Hn.TOL, err
    if topk:
        merr = float(np.abs(mass.cpu().numpy().astype(np.float64) - rmass).max())
        print(f"{g.w.name} step {step}: top-k mass error {merr:.3e}")
        assert merr <= Hn.MASS_TOL, merr
    return err


def test_generator_identical_on_cpu_and_gpu():
    w = W.WORKLOADS["r1-llama-8b"]
    kc, vc = W.kv_values(w, 3, 100, 37, device="cpu")
    kg, vg = W.kv_values(w, 3, 100, 37, device="cuda")
    assert torch.equal(kc, kg.cpu()) and torch.equal(vc, vg.cpu())
    assert torch.equal(W.q_values(w, 5, "cpu"), W.q_values(w, 5, "cuda").cpu())


def test_tiny_workload():
    w = W.WORKLOADS["tiny"]
    g, o = _pair(w)
    g.setup()
    o.setup()
    _check_all(g, o, topk=8)


@pytest.mark.parametrize("name,batch,length", [
    ("r1-llama-8b", 3, 1500),
    ("r1-qwen-14b", 2, 2100),
    ("gpt-oss-20b", 4, None),
    ("churn", 3, None),
])
def test_reduced_configs(name, batch, length):
    """The named shapes with fewer/shorter sequences (several pages per split,
    ragged tails), plus churn steps."""
    base = W.WORKLOADS[name]
    kw = dict(batch=batch, churn_steps=min(base.churn_steps, 20))
    if length is not None:
        kw["lengths"] = ("fixed", length)
    elif base.lengths[0] == "uniform":
        kw["lengths"] = ("uniform", 600, 2500)
    else:
        kw["lengths"] = ("loguniform", 300, 3000)
    w = W.scaled(base, **kw)
    g, o = _pair(w, extra=40)
    g.setup()
    o.setup()
    k = w.topk or 16
    _check_all(g, o, step=0, topk=k)
    for step in range(1, 4):
        g.churn_step()
        o.churn_step()
        _check_all(g, o, step=step, topk=k, codes=(step == 3))


@pytest.mark.parametrize("bits", [(16, 16, 16), (8, 8, 8), (2, 4, 8), (16, 4, 2), (4, 2, 16)])
@pytest.mark.parametrize("d,G", [(64, 32), (128, 64), (128, 32), (64, 64)])
def test_bit_widths_and_shapes(bits, d, G):
    w = W.Workload(name="x", batch=3, num_q_heads=8, num_kv_heads=2, head_dim=d, group_size=G,
                   bits=bits, lengths=("uniform", 40, 700), segments=("geometric", 12),
                   budget=("frac", 0.3), seed=11)
    g, o = _pair(w, extra=10, bits=bits)
    g.setup()
    o.setup()
    _check_all(g, o, topk=5)
    g.churn_step()
    o.churn_step()
    _check_all(g, o, step=1, topk=64)


@pytest.mark.parametrize("hq,hkv", [(1, 1), (2, 2), (5, 1), (8, 1), (40, 8), (6, 3)])
def test_gqa_groups(hq, hkv):
    w = W.Workload(name="x", batch=2, num_q_heads=hq, num_kv_heads=hkv, head_dim=128,
                   group_size=64, lengths=("uniform", 100, 900), budget=("frac", 0.25), seed=5)
    g, o = _pair(w)
    g.setup()
    o.setup()
    _check_all(g, o, topk=3)


def test_no_eviction_dense_16bit():
    """All tokens 16-bit and nothing evicted: plain paged attention."""
    w = W.Workload(name="x", batch=2, num_q_heads=4, num_kv_heads=2, head_dim=64, group_size=32,
                   bits=(16, 16, 16), lengths=("fixed", 333), budget=("fixed", 10 ** 6), seed=2)
    g, o = _pair(w, bits=(16, 16, 16))
    g.setup()
    o.setup()
    _check_all(g, o)


def test_empty_and_fully_evicted_sequences():
    w = W.Workload(name="x", batch=3, num_q_heads=4, num_kv_heads=2, head_dim=64, group_size=32,
                   lengths=("fixed", 50), budget=("fixed", 0), seed=3)
    g, o = _pair(w)
    g.setup()
    o.setup()
    out, mass = g.decode(0, topk=4)
    assert torch.count_nonzero(out) == 0 and torch.count_nonzero(mass) == 0
    _check_all(g, o, topk=4)


@pytest.mark.parametrize("k", [1, 2, 31, 32, 33, 64])
def test_topk_mass_values_of_k(k):
    """k around the candidate-buffer boundaries; long segments force compactions."""
    w = W.Workload(name="x", batch=2, num_q_heads=16, num_kv_heads=2, head_dim=64, group_size=32,
                   lengths=("fixed", 3000), budget=("frac", 0.5), seed=7)
    g, o = _pair(w)
    g.setup()
    o.setup()
    _check_all(g, o, topk=k, codes=False)


@pytest.mark.parametrize("k", [8, 32, 40])
def test_topk_mass_long_pieces_and_tied_logits(k):
    """Enough live pages that every split warp handles about 20 pages of one
    (sequence, kv-head), so its candidate lists fill and are cut back several
    times.  Sequences 0-3 have one key for all tokens: every logit of a head
    ties, no candidate can be dropped by a threshold, and the exact cut must
    keep k of them (mass k / live tokens).  Sequences 4-7 have random keys."""
    from oracle import oracle as O
    from mixed_precision_paged_thinkv_b200.binding import ThinKVCache
    Hq, Hkv, d, G, ns, L = 64, 8, 64, 32, 8, 6144
    g = ThinKVCache(Hq, Hkv, d, G, (8, 4, 2), ns, 512, (ns * L // 16, 16, 16))
    o = O.Oracle(Hq, Hkv, d, G, (8, 4, 2), ns, 512, (ns * L // 16, 16, 16))
    dev = torch.device("cuda")
    gen = torch.Generator().manual_seed(11)
    key = torch.randn(Hkv, d, generator=gen)
    chunk = 512
    for c0 in range(0, L, chunk):
        seq = np.repeat(np.arange(ns), chunk).astype(np.int32)
        pos = np.tile(np.arange(c0, c0 + chunk), ns).astype(np.int32)
        tag = np.zeros(seq.size, np.uint8)
        kk = torch.randn(seq.size, Hkv, d, generator=gen)
        kk[: 4 * chunk] = key                       # sequences 0-3: one key
        kk = kk.half()
        vv = torch.randn(seq.size, Hkv, d, generator=gen).half()
        g.append(torch.as_tensor(seq, device=dev), torch.as_tensor(pos, device=dev),
                 torch.as_tensor(tag, device=dev), kk.to(dev), vv.to(dev))
        assert o.append(seq, pos, tag, kk, vv) == O.OK
    torch.cuda.synchronize()
    assert g.status() == 0
    q = torch.randn(ns, Hq, d, generator=gen).half()
    out, mass = g.decode(torch.arange(ns, dtype=torch.int32, device=dev), q.to(dev), topk=k)
    ref, rmass = o.decode(np.arange(ns, dtype=np.int32), q, topk=k, threads=8)
    torch.cuda.synchronize()
    assert g.status() == 0
    err = Hn.attn_error(out.cpu().numpy(), ref)
    m = mass.cpu().numpy().astype(np.float64)
    merr = float(np.abs(m - rmass).max())
    print(f"long pieces k={k}: attention error {err:.3e}, top-k mass error {merr:.3e}")
    assert err <= Hn.TOL, err
    assert merr <= Hn.MASS_TOL, merr
    assert np.allclose(m[:4], k / L, rtol=1e-3, atol=0), m[:4].min()


@pytest.mark.parametrize("order", [(0, 1, 2), (1, 2, 0), (2, 0, 1), (0, 2, 1)])
def test_eviction_class_orders(order):
    """A non-default class order for eviction (the `order` argument): the
    victims, freed slots and live lists must match the oracle's, through a
    first evict that reaches into every class and churn steps after it."""
    w = W.Workload(name="x", batch=3, num_q_heads=8, num_kv_heads=2, head_dim=128, group_size=64,
                   lengths=("uniform", 300, 900), budget=("frac", 0.2), seed=13)
    g, o = _pair(w, extra=12)
    for call in g.sched.prefill_calls():
        g.append_call(call)
        o.append_call(call)
    dev = torch.device("cuda")
    seqs = torch.arange(w.batch, dtype=torch.int32, device=dev)
    for step in range(4):
        b = g.sched.budgets(g.generated)
        g.cache.evict(seqs, torch.as_tensor(b, device=dev), order=order)
        assert o.o.evict(o.all_seqs, b, order=order) == 0
        _check_all(g, o, step=step, topk=4, codes=(step == 0))
        call = g.sched.one_token_call(g.generated)
        g.append_call(call)
        o.append_call(call)
        g.generated += 1
        o.generated += 1


@pytest.mark.parametrize("scale", [0.02, 0.5])
def test_explicit_softmax_scale(scale):
    """softmax_scale > 0 replaces 1/sqrt(d): a flat (0.02) and a sharp (0.5)
    softmax against the oracle with the same scale."""
    w = W.Workload(name="x", batch=3, num_q_heads=16, num_kv_heads=4, head_dim=64, group_size=32,
                   lengths=("uniform", 200, 1200), budget=("frac", 0.3), seed=17)
    g, o = _pair(w)
    g.setup()
    o.setup()
    torch.cuda.synchronize()
    q = W.q_values(w, 0, device="cuda")
    out, mass = g.cache.decode(g.all_seqs, q, topk=8, softmax_scale=scale)
    ref, rmass = o.o.decode(o.all_seqs, W.q_values(w, 0), softmax_scale=scale, topk=8, threads=8)
    err = Hn.attn_error(out.cpu().numpy(), ref)
    merr = float(np.abs(mass.cpu().numpy().astype(np.float64) - rmass).max())
    print(f"scale {scale}: attention error {err:.3e}, top-k mass error {merr:.3e}")
    assert err <= Hn.TOL and merr <= Hn.MASS_TOL, (err, merr)


def test_decode_shuffled_subset_with_repeated_ids():
    """decode over a permuted subset of the sequences with one id twice: row i
    of the output belongs to seq[i], whatever the order, and a repeated id
    gives the same row twice."""
    w = W.Workload(name="x", batch=6, num_q_heads=16, num_kv_heads=4, head_dim=128, group_size=64,
                   lengths=("uniform", 100, 1500), budget=("frac", 0.25), seed=19)
    g, o = _pair(w)
    g.setup()
    o.setup()
    torch.cuda.synchronize()
    ids = np.array([4, 1, 5, 1, 0], dtype=np.int32)
    qall = W.q_values(w, 3)
    q = qall[[0, 1, 2, 3, 4]].contiguous()           # one query row set per call slot
    out, mass = g.cache.decode(torch.as_tensor(ids, device="cuda"), q.cuda(), topk=6)
    ref, rmass = o.o.decode(ids, q, topk=6, threads=8)
    err = Hn.attn_error(out.cpu().numpy(), ref)
    merr = float(np.abs(mass.cpu().numpy().astype(np.float64) - rmass).max())
    print(f"shuffled subset: attention error {err:.3e}, top-k mass error {merr:.3e}")
    assert err <= Hn.TOL and merr <= Hn.MASS_TOL, (err, merr)
    # the repeated id with the same query gives the same row up to rounding
    # (the two copies' pages fall at different stream-K split points, so
    # their partial sums are merged in different orders)
    q2 = q.clone()
    q2[3] = q2[1]
    out2, _ = g.cache.decode(torch.as_tensor(ids, device="cuda"), q2.cuda())
    assert Hn.attn_error(out2[3:4].cpu().numpy(), out2[1:2].cpu().numpy().astype(np.float64)) <= Hn.TOL


@pytest.mark.parametrize("fmt,bits", [((1, 1, 1), (8, 4, 2)), ((1, 0, 1), (8, 4, 2)),
                                      ((0, 1, 1), (4, 8, 2)), ((1, 1, 0), (2, 8, 4))])
@pytest.mark.parametrize("d,G", [(128, 64), (64, 32)])
def test_float_code_formats(fmt, bits, d, G):
    """The pages' own formats (FP8 E4M3, FP4 E2M1, ternary), alone and mixed
    with integer classes: codes and params bit-exact with the oracle (the
    hardware's E4M3/E2M1 rounding against the formats' definitions), state
    bit-exact, attention and top-k mass within 2e-3, before and after churn."""
    w = W.Workload(name="x", batch=3, num_q_heads=8, num_kv_heads=2, head_dim=d, group_size=G,
                   bits=bits, fmt=fmt, lengths=("uniform", 300, 1200), segments=("geometric", 12),
                   budget=("frac", 0.4), seed=23)
    g, o = _pair(w, extra=10, bits=bits)
    g.setup()
    o.setup()
    _check_all(g, o, topk=8)
    for step in range(1, 3):
        g.churn_step()
        o.churn_step()
        _check_all(g, o, step=step, topk=16)


def test_float_formats_full_size_mixed_state():
    """The r1-llama-8b history kept whole (R/E/T mix at FP8/FP4/ternary), in
    the launch configuration the bench times; sampled sequences against the
    oracle."""
    from mixed_precision_paged_thinkv_b200.runner import WorkloadRun
    w = W.get("r1-llama-8b-mixed-float")
    g = WorkloadRun(w, extra=2)
    g.setup()
    osub = Hn.OracleSubset(w, [0, 7, 15], extra=2)
    osub.setup()
    torch.cuda.synchronize()
    assert g.cache.status() == 0
    snap = g.cache.snapshot()
    ost = osub.o.state()
    for j, s in enumerate(osub.seqs):
        Hn.compare_seq_structure(snap, s, ost, j)
        Hn.compare_codes_by_pos(g.cache, Hn.gpu_live_by_pos(snap, s), osub.o, osub.live_by_pos(j))
    out, _ = g.decode(0)
    ref, _ = osub.decode(0)
    err = Hn.attn_error(out.cpu().numpy()[osub.seqs], ref)
    print(f"r1-llama-8b-mixed-float: attention error {err:.3e}")
    assert err <= Hn.TOL

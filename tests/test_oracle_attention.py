"""Pins of the oracle's decode attention over the paged, mixed-precision cache.

* 16-bit pass-through with no eviction equals textbook fp64 softmax attention
  (numpy) over the raw K/V;
* with eviction and 8/4/2-bit codes, equals numpy attention over the tokens an
  independent set model says are live, dequantised group by group;
* placement invariance: two histories that reach the same live set through
  different slots give bit-identical outputs;
* closed forms: q = 0 gives the mean of the live values and top-k mass
  min(k, n)/n; one dominant key gives its own value and mass ~ 1.
"""
import numpy as np
import pytest

from oracle import oracle as O
from test_oracle_state import SetModel


def _h2f(b):
    return float(np.array([b], dtype=np.uint16).view(np.float16)[0])


def _attn(q, K, V, scale, topk=None):
    """Textbook fp64 softmax attention of one query over rows of K, V."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1]), 0.0
    lg = scale * (K @ q)
    p = np.exp(lg - lg.max())
    p /= p.sum()
    mass = None
    if topk:
        mass = 1.0 if K.shape[0] <= topk else np.sort(p)[::-1][:topk].sum()
    return p @ V, mass


def _deq_rows(x, bits, G):
    """Dequantise rows of fp16 x (shape [n, d]) group by group with the oracle quantiser."""
    if bits == 16:
        return x.astype(np.float64)
    out = np.zeros(x.shape, dtype=np.float64)
    for i in range(x.shape[0]):
        for g in range(0, x.shape[1], G):
            c, s, z = O.quantize_group(x[i, g:g + G], bits)
            out[i, g:g + G] = _h2f(z) + c.astype(np.float64) * _h2f(s)
    return out


def _history(rng, ns, steps, H, d, evict=True):
    """Random append/evict history; returns ops and per-sequence token data."""
    ops, nextpos = [], [0] * ns
    data = {s: {} for s in range(ns)}          # pos -> (tag, k[H,d], v[H,d])
    for op in range(steps):
        if rng.random() < 0.65 or not evict:
            S, P, T, K, V = [], [], [], [], []
            for s in rng.permutation(ns)[:rng.integers(1, ns + 1)]:
                for _ in range(int(rng.integers(1, 20))):
                    t = int(rng.choice(3, p=[.3, .5, .2]))
                    k = (rng.standard_normal((H, d)) * rng.choice([1, 1, 8])).astype(np.float16)
                    v = rng.standard_normal((H, d)).astype(np.float16)
                    S.append(int(s)); P.append(nextpos[s]); T.append(t); K.append(k); V.append(v)
                    data[int(s)][nextpos[s]] = (t, k, v)
                    nextpos[s] += 1
            ops.append(("a", S, P, T, np.stack(K), np.stack(V)))
        else:
            seqs = [int(x) for x in rng.permutation(ns)[:rng.integers(1, ns + 1)]]
            ops.append(("e", seqs, [int(rng.integers(0, 25)) for _ in seqs]))
    return ops, data


def _run(o, model, ops):
    for op in ops:
        if op[0] == "a":
            assert o.append(*op[1:]) == O.OK
            model.append(op[1], op[2], op[3])
        else:
            assert o.evict(op[1], op[2]) == O.OK
            model.evict(op[1], op[2])


@pytest.mark.parametrize("gq", [1, 4])
def test_dense_16bit_no_eviction_equals_textbook_attention(gq):
    rng = np.random.default_rng(gq)
    ns, H, d = 3, 2, 64
    o = O.Oracle(H * gq, H, d, 32, (16, 16, 16), ns, 20, (40, 40, 40))
    model = SetModel(ns)
    ops, data = _history(rng, ns, 12, H, d, evict=False)
    _run(o, model, ops)
    q = rng.standard_normal((ns, H * gq, d)).astype(np.float16)
    out, mass = o.decode(list(range(ns)), q, topk=5)
    scale = 1 / np.sqrt(d)
    for s in range(ns):
        poss = sorted(data[s])
        for hq in range(H * gq):
            h = hq // gq
            K = np.stack([data[s][p][1][h] for p in poss]).astype(np.float64)
            V = np.stack([data[s][p][2][h] for p in poss]).astype(np.float64)
            ref, m = _attn(q[s, hq].astype(np.float64), K, V, scale, topk=5)
            np.testing.assert_allclose(out[s, hq], ref, rtol=1e-12, atol=1e-14)
            assert abs(mass[s, hq] - m) < 1e-12


@pytest.mark.parametrize("bits", [(8, 4, 2), (16, 8, 2), (4, 4, 4)])
def test_mixed_precision_with_eviction_equals_attention_over_live_set(bits):
    rng = np.random.default_rng(sum(bits))
    ns, H, d, G, gq = 3, 2, 64, 32, 2
    o = O.Oracle(H * gq, H, d, G, bits, ns, 30, (60, 60, 60))
    model = SetModel(ns)
    ops, data = _history(rng, ns, 30, H, d)
    _run(o, model, ops)
    q = rng.standard_normal((ns, H * gq, d)).astype(np.float16)
    scale = 0.37
    out, mass = o.decode(list(range(ns)), q, softmax_scale=scale, topk=3)
    for s in range(ns):
        poss = sorted(model.live[s])
        for hq in range(H * gq):
            h = hq // gq
            if not poss:
                assert not out[s, hq].any() and mass[s, hq] == 0.0
                continue
            K = np.concatenate([_deq_rows(data[s][p][1][h:h + 1], bits[data[s][p][0]], G) for p in poss])
            V = np.concatenate([_deq_rows(data[s][p][2][h:h + 1], bits[data[s][p][0]], G) for p in poss])
            ref, m = _attn(q[s, hq].astype(np.float64), K, V, scale, topk=3)
            np.testing.assert_allclose(out[s, hq], ref, rtol=1e-11, atol=1e-13)
            assert abs(mass[s, hq] - m) < 1e-12


def test_placement_invariance():
    """Same live tokens reached through different slots -> identical outputs."""
    rng = np.random.default_rng(5)
    H, d, G = 2, 64, 32
    n = 40
    tags = rng.choice(3, size=n, p=[.3, .5, .2]).astype(np.uint8)
    K = rng.standard_normal((n, H, d)).astype(np.float16)
    V = rng.standard_normal((n, H, d)).astype(np.float16)
    q = rng.standard_normal((1, 4, d)).astype(np.float16)
    # history A: seq 0 appends tokens 0..39 in one call
    a = O.Oracle(4, H, d, G, (8, 4, 2), 2, 20, (40, 40, 40))
    assert a.append([0] * n, list(range(n)), tags, K, V) == O.OK
    # history B: seq 1 first gets dummy tokens that are then evicted (so its
    # slots are reused in a different order), and the real tokens arrive in
    # several calls interleaved with another sequence
    b = O.Oracle(4, H, d, G, (8, 4, 2), 2, 20, (40, 40, 40))
    dummy_t = rng.choice(3, size=25).astype(np.uint8)
    dk = rng.standard_normal((25, H, d)).astype(np.float16)
    assert b.append([1] * 25, list(range(25)), dummy_t, dk, dk) == O.OK
    assert b.evict([1], [0]) == O.OK
    for lo, hi in ((0, 7), (7, 23), (23, 40)):
        other_t = rng.choice(3, size=3).astype(np.uint8)
        seqs = [0] * 3 + [1] * (hi - lo)
        pos = [1000 + lo, 1001 + lo, 1002 + lo] + list(range(100 + lo, 100 + hi))
        assert b.append(seqs, pos, np.concatenate([other_t, tags[lo:hi]]),
                        np.concatenate([dk[:3], K[lo:hi]]),
                        np.concatenate([dk[:3], V[lo:hi]])) == O.OK
    oa, ma = a.decode([0], q, topk=7)
    ob, mb = b.decode([1], q, topk=7)
    assert np.array_equal(oa, ob)
    assert np.array_equal(ma, mb)


def test_closed_forms():
    rng = np.random.default_rng(9)
    H, d, G, n = 1, 64, 32, 37
    o = O.Oracle(2, H, d, G, (8, 4, 2), 1, 10, (10, 10, 10))
    tags = rng.choice(3, size=n).astype(np.uint8)
    K = rng.standard_normal((n, H, d)).astype(np.float16)
    V = rng.standard_normal((n, H, d)).astype(np.float16)
    assert o.append([0] * n, list(range(n)), tags, K, V) == O.OK
    # q = 0: uniform attention -> mean of the dequantised values; mass min(k,n)/n
    q = np.zeros((1, 2, d), dtype=np.float16)
    out, mass = o.decode([0], q, topk=5)
    Vd = np.concatenate([_deq_rows(V[i, 0:1], (8, 4, 2)[tags[i]], G) for i in range(n)])
    np.testing.assert_allclose(out[0, 0], Vd.mean(axis=0), rtol=1e-12, atol=1e-14)
    assert abs(mass[0, 0] - 5 / n) < 1e-14
    # one dominant key: output -> its value, mass -> 1
    K2 = K.copy()
    K2[:] = 0
    K2[13] = 8.0
    o2 = O.Oracle(2, H, d, G, (8, 8, 8), 1, 10, (10, 10, 10))
    assert o2.append([0] * n, list(range(n)), tags, K2, V) == O.OK
    q2 = np.full((1, 2, d), 8.0, dtype=np.float16)
    out2, mass2 = o2.decode([0], q2, topk=1)
    v13 = _deq_rows(V[13, 0:1], 8, G)[0]
    np.testing.assert_allclose(out2[0, 0], v13, rtol=1e-9, atol=1e-9)
    assert mass2[0, 0] > 1 - 1e-9
    # k >= n -> mass exactly 1
    _, m3 = o.decode([0], rng.standard_normal((1, 2, d)).astype(np.float16), topk=n)
    assert np.all(m3 == 1.0)

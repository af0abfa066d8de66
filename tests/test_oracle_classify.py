"""Pins of the oracle's thought classifier (mechanism only): hand-worked
examples, the ordering T > R > E by attention sparsity, and the top-k masses
that the oracle's own decode produces for attention of known sparsity."""
import os

import numpy as np

from oracle import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    rows = []
    for line in open(os.path.join(HERE, "golden", "classify_examples.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        th, ms, tag = [x.strip() for x in line.split("|")]
        tt, tr = [float.fromhex(x) for x in th.split()]
        masses = np.array([float.fromhex(x) for x in ms.split()], dtype=np.float32)
        rows.append((tt, tr, masses, int(tag)))
    return rows


def test_hand_worked_examples():
    rows = _golden()
    assert len(rows) == 9
    for k, (tt, tr, m, tag) in enumerate(rows):
        got = O.classify(m[None, :], tt, tr)
        assert int(got[0]) == tag, (k + 1, int(got[0]), tag)


def test_order_and_monotonicity():
    """Raising every head's mass never makes a sequence less sparse in the
    tags' order E < R < T; permuting sequences permutes their tags."""
    rng = np.random.default_rng(3)
    rank = {1: 0, 0: 1, 2: 2}                      # E < R < T
    m = rng.random((500, 16)).astype(np.float32)
    a = O.classify(m, 0.7, 0.4)
    b = O.classify(np.minimum(m + np.float32(0.05), np.float32(1)), 0.7, 0.4)
    assert all(rank[int(y)] >= rank[int(x)] for x, y in zip(a, b))
    perm = rng.permutation(500)
    assert np.array_equal(O.classify(m[perm], 0.7, 0.4), a[perm])
    assert set(np.unique(a).tolist()) == {0, 1, 2}


def test_tags_from_decode_masses_of_known_sparsity():
    """The oracle's decode on a state of known attention sparsity: every key
    equal gives each head a mass of exactly k / n (dense attention -> E); one
    key aligned with and far larger than the others gives a mass near 1
    (sparse -> T)."""
    Hq, Hkv, d, G, n = 4, 2, 64, 32, 256
    o = O.Oracle(Hq, Hkv, d, G, (16, 16, 16), 2, 64, (64, 1, 1))
    rng = np.random.default_rng(5)
    q = rng.standard_normal((2, Hq, d)).astype(np.float16)
    k = np.zeros((2 * n, Hkv, d), dtype=np.float16)
    k[:n] = rng.standard_normal((Hkv, d)).astype(np.float16)      # seq 0: one key for all
    k[n:] = (0.01 * rng.standard_normal((n, Hkv, d))).astype(np.float16)
    k[n + 7] = (np.repeat(q[1].astype(np.float32).reshape(Hkv, 2, d).sum(1, keepdims=False)[:, None, :],
                          1, axis=1)[:, 0, :] * 4).astype(np.float16)   # seq 1: one dominant key
    v = rng.standard_normal((2 * n, Hkv, d)).astype(np.float16)
    seq = np.repeat(np.arange(2, dtype=np.int32), n)
    pos = np.tile(np.arange(n, dtype=np.int32), 2)
    assert o.append(seq, pos, np.zeros(2 * n, np.uint8), k, v) == O.OK
    _, mass = o.decode(np.arange(2, dtype=np.int32), q, topk=8, threads=2)
    assert np.allclose(mass[0], 8 / n, rtol=0, atol=1e-12)
    assert mass[1].min() > 0.99
    tags = O.classify(mass.astype(np.float32), 0.9, 0.2)
    assert tags.tolist() == [1, 2]

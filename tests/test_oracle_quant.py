"""Pins of the oracle's group quantiser (thought-adaptive precision, TBQ).

* hand-worked examples (tests/golden/quant_examples.txt);
* the error bound |x - (zero + code*scale)| <= scale * (1/2 + 2^-14);
* brute force: the code is the fp64-nearest level (ties to the even code),
  except within 2^-14 of a tie, where the spec's two fp32 roundings decide;
* range: zero <= min(x) and zero + (2^b - 1) * scale >= max(x).
"""
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from mixed_precision_paged_thinkv_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_examples.txt")


def _h2f(bits: int) -> float:
    return float(np.array([bits], dtype=np.uint16).view(np.float16)[0])


def _cases():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        b, xs, z, s, codes = [p.strip() for p in line.split("|")]
        out.append((int(b), [float(t) for t in xs.split()], int(z, 16), int(s, 16),
                    [int(t) for t in codes.split()]))
    return out


@pytest.mark.parametrize("bits,xs,zero,scale,codes", _cases())
def test_hand_worked_examples(bits, xs, zero, scale, codes):
    x = np.array(xs, dtype=np.float16)
    assert np.array_equal(x.astype(np.float64), np.array(xs)), "inputs must be fp16-exact"
    c, s, z = O.quantize_group(x, bits)
    assert z == zero
    assert s == scale
    assert c.tolist() == codes


def _groups(bits, G, n, seed):
    rng = np.random.default_rng(seed)
    kinds = [
        rng.standard_normal((n, G)),
        rng.standard_normal((n, G)) * 8.0,                       # outlier-scale groups
        rng.uniform(-1e-3, 1e-3, (n, G)),                        # tiny ranges (subnormal scales)
        rng.uniform(100, 30000, (n, G)) * rng.choice([-1, 1], (n, 1)),
        np.round(rng.uniform(0, 2 ** bits - 1, (n, G))) * 0.25,  # values on a level grid
    ]
    x = np.concatenate(kinds).astype(np.float16)
    x[0, :] = x[0, 0]                                            # one constant group
    return x


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("G", [32, 64])
def test_bound_range_and_brute_force(bits, G):
    x = _groups(bits, G, 300, seed=bits * 100 + G)
    levels = 2 ** bits - 1
    for row in x:
        c, sb, zb = O.quantize_group(row, bits)
        s, z = _h2f(sb), _h2f(zb)
        xd = row.astype(np.float64)
        deq = z + c.astype(np.float64) * s
        # range
        assert z <= xd.min()
        assert z + levels * s >= xd.max()
        if s == 0.0:
            assert xd.min() == xd.max() and not c.any()
            continue
        # error bound
        assert np.all(np.abs(xd - deq) <= s * (0.5 + 2.0 ** -14))
        # brute force over every level in fp64; ties -> even code
        t = (xd - z) / s
        cand = np.arange(levels + 1, dtype=np.float64)
        err = np.abs(xd[:, None] - (z + cand[None, :] * s))
        best = err.min(axis=1, keepdims=True)
        is_best = err <= best * (1 + 1e-15)
        brute = np.array([
            (lambda idx: idx[(idx % 2) == 0][0] if len(idx) > 1 and (idx % 2 == 0).any() else idx[0])(
                np.flatnonzero(r)) for r in is_best])
        near_tie = np.abs(t - np.floor(t) - 0.5) < 2.0 ** -14
        mism = (brute != c) & ~near_tie
        assert not mism.any(), (row[mism], c[mism], brute[mism])


def test_generator_data_obeys_bound():
    """On the workload generator's K/V (with x8 outlier channels)."""
    w = W.WORKLOADS["tiny"]
    k, v = W.kv_values(w, 0, 0, 64)
    for t in (k, v):
        for row in t.reshape(-1, w.group_size).numpy():
            for bits in (2, 4, 8):
                c, sb, zb = O.quantize_group(row, bits)
                s, z = _h2f(sb), _h2f(zb)
                deq = z + c.astype(np.float64) * s
                assert np.all(np.abs(row.astype(np.float64) - deq) <= s * (0.5 + 2.0 ** -14))


def test_more_bits_never_worse_on_average():
    """Precision is ordered by bit width (R > E > T): mean error shrinks with b."""
    x = _groups(8, 64, 100, seed=7)[:200]
    errs = []
    for bits in (2, 4, 8):
        e = 0.0
        for row in x:
            c, sb, zb = O.quantize_group(row, bits)
            e += np.abs(row.astype(np.float64) - (_h2f(zb) + c * _h2f(sb))).mean()
        errs.append(e)
    assert errs[0] > errs[1] > errs[2]

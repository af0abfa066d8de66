"""Pins of the oracle's float code formats (the explainer's TBQ names FP8,
NVFP4 and ternary): the E4M3 value table against torch's float8_e4m3fn, the
E2M1 table against its eight published magnitudes, rounding against brute
force over the tables (nearest, ties to even, saturating), hand-worked groups
for each format, the error bound, and attention over float-coded states
against textbook fp64 attention over the dequantised values."""
import numpy as np
import pytest
import torch

from oracle import oracle as O

E2M1_MAGNITUDES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e4m3_table_matches_torch_float8():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    ours = np.array([O.e4m3_value(c) for c in range(256)])
    fin = np.isfinite(ref)
    assert np.array_equal(np.isnan(ours), ~fin)
    assert np.array_equal(ours[fin], ref[fin].astype(np.float64))
    assert O.e4m3_value(0x7E) == 448.0 and O.e4m3_value(0x08) == 2.0 ** -6
    assert O.e4m3_value(0x01) == 2.0 ** -9


def test_e2m1_table():
    ours = [O.e2m1_value(c) for c in range(16)]
    assert ours[:8] == E2M1_MAGNITUDES
    assert ours[8:] == [-m for m in E2M1_MAGNITUDES]


def _brute(vals, codes, a):
    """nearest finite value, ties to the even code, saturating (magnitudes)."""
    d = np.abs(vals[None, :] - a[:, None])
    best = d.min(axis=1, keepdims=True)
    cand = np.where(d == best, codes[None, :], 10 ** 6)
    even = np.where((cand % 2 == 0) & (cand < 10 ** 6), cand, 10 ** 6)
    pick = np.where(even.min(axis=1) < 10 ** 6, even.min(axis=1), cand.min(axis=1))
    return np.where(a >= vals.max(), codes[np.argmax(vals)], pick)


def test_e4m3_rounding_brute_force_and_torch():
    rng = np.random.default_rng(0)
    codes = np.arange(0x7F)                       # finite non-negative codes
    vals = np.array([O.e4m3_value(c) for c in codes])
    a = np.concatenate([np.abs(rng.standard_normal(3000)) * 10.0 ** rng.integers(-4, 3, 3000),
                        (vals[:-1] + vals[1:]) / 2, vals, [448.0, 463.9, 464.0, 1e6]]).astype(np.float32)
    ours = np.array([O.e4m3_from_f32(float(x)) for x in a])
    assert np.array_equal(ours, _brute(vals, codes, a.astype(np.float64)))
    inr = a < 464.0                                # torch does not saturate
    tq = torch.as_tensor(a[inr]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours[inr], tq)
    neg = np.array([O.e4m3_from_f32(-float(x)) for x in a[:200]])
    assert np.array_equal(neg, ours[:200] | 0x80)


def test_e2m1_rounding_brute_force():
    rng = np.random.default_rng(1)
    codes = np.arange(8)
    vals = np.array(E2M1_MAGNITUDES)
    a = np.concatenate([rng.random(3000) * 8, (vals[:-1] + vals[1:]) / 2, vals, [7.0, 100.0]]).astype(np.float32)
    ours = np.array([O.e2m1_from_f32(float(x)) for x in a])
    assert np.array_equal(ours, _brute(vals, codes, a.astype(np.float64)))
    # the ties, worked by hand: 0.25 -> 0, 0.75 -> 1.0, 1.25 -> 1.0, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    assert [O.e2m1_value(O.e2m1_from_f32(t)) for t in ties] == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]


def _h(xs):
    return np.array(xs, dtype=np.float16)


def test_hand_worked_groups():
    # FP8: amax 3.5 -> scale = 3.5/448 = 2^-7 exactly; x/s = 448, -128, 0, 38.4 -> 0x7E,
    # 0xF0 (-(2^7): exponent 14, mantissa 0), 0x00, 38.4 -> 40 (quantum 4 in [32, 64),
    # 9.6 -> 10) = 1.25 * 2^5 -> exponent 12, mantissa 2 -> 0x62
    c, s, z = O.quantize_group(_h([3.5, -1.0, 0.0, 0.30004883]), 8, fmt=1)
    assert c.tolist() == [0x7E, 0xF0, 0x00, 0x62] and s == 0x2000 and z == 0
    # FP4: amax 6 -> scale 1; 6 -> 7, -3 -> 8 | 5 = 13, 1.2 -> 1.0 (code 2), 0.2 -> 0
    c, s, z = O.quantize_group(_h([6.0, -3.0, 1.2, 0.2]), 4, fmt=1)
    assert c.tolist() == [7, 13, 2, 0] and s == 0x3C00 and z == 0
    # ternary: amax 1 -> scale 1, zero -1; x/s = 1, -0.5, 0.25, -1 -> rint_even 1, 0, 0, -1
    # -> codes (+1) 2, 1, 1, 0
    c, s, z = O.quantize_group(_h([1.0, -0.5, 0.25, -1.0]), 2, fmt=1)
    assert c.tolist() == [2, 1, 1, 0] and s == 0x3C00 and z == 0xBC00
    # a zero group: scale 0, the code of 0 everywhere
    for b, zc in ((8, 0), (4, 0), (2, 1)):
        c, s, z = O.quantize_group(_h([0.0] * 8), b, fmt=1)
        assert set(c.tolist()) == {zc} and s == 0


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_float_format_error_bound(bits):
    """No code saturates below the group's maximum, and |x - deq| is at most
    half the format's spacing around x/scale (times scale); ternary: at most
    scale/2."""
    rng = np.random.default_rng(bits)
    for _ in range(300):
        x = (rng.standard_normal(64) * 10.0 ** rng.integers(-3, 3)).astype(np.float16)
        c, s, z = O.quantize_group(x, bits, fmt=1)
        sf = float(np.array([s], np.uint16).view(np.float16)[0])
        xf = x.astype(np.float64)
        if bits == 2:
            deq = sf * (c.astype(np.float64) - 1)
            assert np.all(np.abs(xf - deq) <= sf / 2 + 1e-12)
            continue
        val = O.e4m3_value if bits == 8 else O.e2m1_value
        deq = np.array([sf * val(int(k)) for k in c])
        table = np.array(sorted({abs(val(k)) for k in range(256 if bits == 8 else 16)
                                 if np.isfinite(val(k))}))
        t = np.abs(xf / sf)
        assert t.max() <= table.max() * (1 + 1e-12)
        i = np.clip(np.searchsorted(table, t), 1, len(table) - 1)
        gap = table[i] - table[i - 1]
        assert np.all(np.abs(xf - deq) <= sf * gap / 2 + 1e-12)


@pytest.mark.parametrize("bits", [(8, 4, 2), (4, 2, 8), (2, 8, 4)])
def test_attention_over_float_codes_is_attention_over_dequantised_values(bits):
    """The oracle's decode with float formats equals textbook fp64 softmax
    attention over scale * value(code) (ternary: scale * (code - 1))."""
    H, d, G, n = 2, 64, 32, 300
    rng = np.random.default_rng(5)
    o = O.Oracle(4, H, d, G, bits, 1, 64, (40, 40, 40), fmt=(1, 1, 1))
    tag = rng.integers(0, 3, n).astype(np.uint8)
    k = rng.standard_normal((n, H, d)).astype(np.float16)
    v = rng.standard_normal((n, H, d)).astype(np.float16)
    assert o.append(np.zeros(n, np.int32), np.arange(n, dtype=np.int32), tag, k, v) == O.OK
    q = rng.standard_normal((1, 4, d)).astype(np.float16)
    out, _ = o.decode(np.zeros(1, np.int32), q)
    # dequantise token by token from the group quantiser directly
    kh = np.zeros((n, H, d))
    vh = np.zeros((n, H, d))
    for i in range(n):
        b = bits[tag[i]]
        for h in range(H):
            for arr, dst in ((k, kh), (v, vh)):
                for g0 in range(0, d, G):
                    c, s, z = O.quantize_group(arr[i, h, g0:g0 + G], b, fmt=1)
                    sf = float(np.array([s], np.uint16).view(np.float16)[0])
                    if b == 2:
                        dst[i, h, g0:g0 + G] = sf * (c.astype(np.float64) - 1)
                    else:
                        val = O.e4m3_value if b == 8 else O.e2m1_value
                        dst[i, h, g0:g0 + G] = [sf * val(int(x)) for x in c]
    for hq in range(4):
        h = hq // 2
        lg = kh[:, h, :] @ q[0, hq].astype(np.float64) / np.sqrt(d)
        p = np.exp(lg - lg.max())
        p /= p.sum()
        assert np.allclose(out[0, hq], p @ vh[:, h, :], rtol=0, atol=1e-12)

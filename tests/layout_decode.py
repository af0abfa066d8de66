"""Decode page-head blocks of libthinkv's pools into natural arrays (numpy).

Written from the layout documented in include/thinkv.h, independently of the
CUDA sources, so that the GPU's packed codes can be compared one by one with
the oracle's natural [slot][channel] codes:

  K codes: lane l = 4*gid + tid owns d*b/16 bytes; for group gr and r in {0,1}
    a piece of G*b/32 bytes holds slot gid + 8r, channels gr*G + tid*G/4 + e;
  V codes: lane l owns words (P, q); word (P, q) has slot 2*tid + 8P in its low
    half and slot 2*tid + 8P + 1 in its high half, element k of each half being
    channel 16*(e//2) + gid + 8*(e%2), e = q*16/b + k;
  params are [group][slot][scale, zero] fp16;
  inside a 32-bit word (or a 16-bit piece) even channels fill the low half and
  odd channels the high half, little-endian;
  the lanes' portions (d*b/16 bytes each) are interleaved in chunks of
  u = min(16, d*b/16) bytes: byte o of lane l sits at (o // u)*32*u + l*u + o % u
  of the K (or V) code region.
"""
from functools import lru_cache

import numpy as np

PAGE = 16


@lru_cache(maxsize=None)
def _maps(d: int, G: int, b: int):
    """(byte offset, bit shift) of every (slot, channel) code, for K and for V."""
    lane_bytes = d * b // 16
    u = min(16, lane_bytes)

    def lpos(lane, o):                      # byte o of the lane's portion
        return (o // u) * 32 * u + lane * u + o % u

    kb = np.zeros((PAGE, d), dtype=np.int64)
    ks = np.zeros((PAGE, d), dtype=np.int64)
    vb = np.zeros((PAGE, d), dtype=np.int64)
    vs = np.zeros((PAGE, d), dtype=np.int64)
    ng = d // G
    pb = G * b // 32                      # piece bytes
    for lane in range(32):
        gid, tid = lane // 4, lane % 4
        # K pieces
        for gr in range(ng):
            for r in range(2):
                slot = gid + 8 * r
                off = (gr * 2 + r) * pb
                for e in range(G // 4):
                    ch = gr * G + tid * (G // 4) + e
                    if b == 16:
                        kb[slot, ch] = lpos(lane, off + 2 * e)
                        ks[slot, ch] = 0
                        continue
                    piece_bits = pb * 8
                    word_bits = min(32, piece_bits)
                    m = word_bits // b             # codes per word (or per 16-bit piece)
                    wi, el = divmod(e, m)
                    p = el // 2 if el % 2 == 0 else m // 2 + el // 2
                    bit = wi * word_bits + p * b
                    kb[slot, ch] = lpos(lane, off + bit // 8)
                    ks[slot, ch] = bit % 8
        # V words
        Q = d * b // 128 if b < 16 else d // 8
        per = 16 // b if b < 16 else 1
        for P in range(2):
            for q in range(Q):
                woff = (P * Q + q) * 4
                for half in range(2):
                    slot = 2 * tid + 8 * P + half
                    for k in range(per):
                        e = q * per + k
                        ch = 16 * (e // 2) + gid + 8 * (e % 2)
                        bit = half * 16 + k * (b if b < 16 else 16)
                        vb[slot, ch] = (2 * d * b if b < 16 else 32 * d) + lpos(lane, woff + bit // 8)
                        vs[slot, ch] = bit % 8
    return kb, ks, vb, vs


def decode_blocks(blocks: np.ndarray, d: int, G: int, b: int):
    """blocks: uint8 [..., page_head_bytes].  Returns (kcodes, vcodes, kparams, vparams)
    with codes [..., 16, d] (uint8, or uint16 raw fp16 bits for b == 16) and params
    [..., 16, d//G, 2] uint16 (None for b == 16)."""
    kb, ks, vb, vs = _maps(d, G, b)
    if b == 16:
        def raw(bo):
            lo = blocks[..., bo].astype(np.uint16)
            hi = blocks[..., bo + 1].astype(np.uint16)
            return lo | (hi << 8)
        return raw(kb), raw(vb), None, None
    mask = (1 << b) - 1
    kc = ((blocks[..., kb] >> ks) & mask).astype(np.uint8)
    vc = ((blocks[..., vb] >> vs) & mask).astype(np.uint8)
    ng = d // G
    po = 4 * d * b
    # params are stored [group][slot][scale, zero]; returned as [slot][group][2]
    kp = blocks[..., po:po + 64 * ng].copy().view(np.uint16).reshape(blocks.shape[:-1] + (ng, PAGE, 2))
    vp = blocks[..., po + 64 * ng:po + 128 * ng].copy().view(np.uint16).reshape(blocks.shape[:-1] + (ng, PAGE, 2))
    return kc, vc, np.swapaxes(kp, -3, -2), np.swapaxes(vp, -3, -2)

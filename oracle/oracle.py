"""Python handle on the CPU oracle (``thinkv_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``.  The CUDA library never
imports, links or calls anything here, and nothing here touches a GPU.

``build()`` compiles the C oracle with gcc (no fast-math, no FP contraction)
into ``oracle/_build/``; ``Oracle`` wraps one oracle state.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
BUILD_DIR = os.path.join(HERE, "_build")
SRC = os.path.join(HERE, "thinkv_oracle.c")
HDR = os.path.join(HERE, "thinkv_oracle.h")
LIB = os.path.join(BUILD_DIR, "libthinkv_oracle.so")

OK, ERR_INVALID, ERR_OUT_OF_PAGES, ERR_OUT_OF_BLOCKS = 0, 1, 2, 3
PAGE = 16

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library (idempotent)."""
    os.makedirs(BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(LIB) or
             os.path.getmtime(LIB) < max(os.path.getmtime(SRC), os.path.getmtime(HDR)))
    if force or stale:
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fexcess-precision=standard", "-fno-fast-math", "-fopenmp",
               SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


class _Layout(C.Structure):
    _fields_ = [("num_q_heads", C.c_int32), ("num_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("page_size", C.c_int32),
                ("group_size", C.c_int32), ("bits", C.c_int32 * 3),
                ("max_seqs", C.c_int32), ("max_blocks_per_seq", C.c_int32),
                ("pool_pages", C.c_int32 * 3), ("fmt", C.c_int32 * 3)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            P = C.c_void_p
            L.or_create.restype = P
            L.or_create.argtypes = [C.POINTER(_Layout)]
            L.or_destroy.argtypes = [P]
            L.or_append.argtypes = [P, C.c_int32, P, P, P, P, P]
            L.or_evict.argtypes = [P, C.c_int32, P, P, P]
            L.or_decode.argtypes = [P, C.c_int32, P, P, C.c_double, C.c_int32, P, P, C.c_int32]
            for f in ("or_f16_round_down", "or_f16_round_up", "or_f16_round_nearest"):
                getattr(L, f).argtypes = [C.c_float]
                getattr(L, f).restype = C.c_uint16
            L.or_f16_to_f32.argtypes = [C.c_uint16]
            L.or_f16_to_f32.restype = C.c_float
            L.or_f16_round_array.argtypes = [P, C.c_int64, C.c_int32, P]
            L.or_quantize_group.argtypes = [P, C.c_int32, C.c_int32, P, P, P]
            L.or_quantize_group_fmt.argtypes = [P, C.c_int32, C.c_int32, C.c_int32, P, P, P]
            for f in ("or_e4m3_value", "or_e2m1_value"):
                getattr(L, f).argtypes = [C.c_uint8]
                getattr(L, f).restype = C.c_double
            for f in ("or_e4m3_from_f32", "or_e2m1_from_f32"):
                getattr(L, f).argtypes = [C.c_float]
                getattr(L, f).restype = C.c_uint8
            L.or_classify.argtypes = [C.c_int32, C.c_int32, P, C.c_float, C.c_float, P]
            L.or_tbe.argtypes = [P, C.c_int32, P, P, P, C.c_int32, P]
            L.or_evict_slots.argtypes = [P, C.c_int32, P, P, P]
            L.or_compact.argtypes = [P, P, C.c_int32, P]
            for f in ("or_codes", "or_params", "or_slot_pos"):
                getattr(L, f).argtypes = [P, C.c_int]
                getattr(L, f).restype = P
            for f in ("or_table", "or_num_blocks", "or_free_slots", "or_free_top", "or_fifo",
                      "or_fifo_head", "or_fifo_tail", "or_live_count", "or_live_list",
                      "or_live_index", "or_num_live", "or_page_bump", "or_seg", "or_nseg"):
                getattr(L, f).argtypes = [P]
                getattr(L, f).restype = P
            _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _u16(x) -> np.ndarray:
    """fp16 data (numpy float16 or torch tensor) as contiguous uint16 bits."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().contiguous().numpy()
    a = np.ascontiguousarray(x)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16
    return a


# -- building blocks (pin tests) -------------------------------------------- #
def f16_round_down(x: float) -> int:
    return int(lib().or_f16_round_down(C.c_float(x)))


def f16_round_up(x: float) -> int:
    return int(lib().or_f16_round_up(C.c_float(x)))


def f16_round_nearest(x: float) -> int:
    return int(lib().or_f16_round_nearest(C.c_float(x)))


def f16_round_array(x: np.ndarray, mode: str) -> np.ndarray:
    """Round fp32 values to fp16 bit patterns: mode 'down', 'up' or 'nearest'."""
    xs = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(xs.shape, dtype=np.uint16)
    m = {"down": 0, "up": 1, "nearest": 2}[mode]
    lib().or_f16_round_array(_ptr(xs), xs.size, m, _ptr(out))
    return out


def quantize_group(x, bits: int, fmt: int = 0):
    """Quantise one group of fp16 values: returns (codes uint8, scale bits, zero bits)."""
    xs = _u16(x)
    G = xs.shape[0]
    codes = np.zeros(G, dtype=np.uint8)
    s = np.zeros(1, dtype=np.uint16)
    z = np.zeros(1, dtype=np.uint16)
    if fmt:
        lib().or_quantize_group_fmt(_ptr(xs), G, bits, fmt, _ptr(codes), _ptr(s), _ptr(z))
    else:
        lib().or_quantize_group(_ptr(xs), G, bits, _ptr(codes), _ptr(s), _ptr(z))
    return codes, int(s[0]), int(z[0])


def e4m3_value(code: int) -> float:
    return float(lib().or_e4m3_value(int(code)))


def e2m1_value(code: int) -> float:
    return float(lib().or_e2m1_value(int(code)))


def e4m3_from_f32(x: float) -> int:
    return int(lib().or_e4m3_from_f32(float(x)))


def e2m1_from_f32(x: float) -> int:
    return int(lib().or_e2m1_from_f32(float(x)))


def classify(mass, theta_t: float, theta_r: float) -> np.ndarray:
    """R/E/T tags (uint8 [n]) from top-k masses (float32 [n, hq])."""
    m = np.ascontiguousarray(mass, dtype=np.float32)
    n, hq = m.shape
    tags = np.zeros(n, dtype=np.uint8)
    lib().or_classify(n, hq, _ptr(m), C.c_float(theta_t), C.c_float(theta_r), _ptr(tags))
    return tags


# -- one oracle cache ---------------------------------------------------------- #
class Oracle:
    """One oracle state with the given geometry."""

    def __init__(self, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 group_size: int, bits: Sequence[int], max_seqs: int,
                 max_blocks_per_seq: int, pool_pages: Sequence[int],
                 fmt: Sequence[int] = (0, 0, 0)):
        self.Hq, self.H, self.d, self.G = num_q_heads, num_kv_heads, head_dim, group_size
        self.fmt = tuple(int(f) for f in fmt)
        self.bits = tuple(int(b) for b in bits)
        self.max_seqs, self.max_blocks = max_seqs, max_blocks_per_seq
        self.pool_pages = tuple(int(p) for p in pool_pages)
        lay = _Layout(num_q_heads, num_kv_heads, head_dim, PAGE, group_size,
                      (C.c_int32 * 3)(*self.bits), max_seqs, max_blocks_per_seq,
                      (C.c_int32 * 3)(*self.pool_pages), (C.c_int32 * 3)(*self.fmt))
        self._lay = lay
        self._h = lib().or_create(C.byref(lay))
        if not self._h:
            raise ValueError("oracle: invalid layout or out of host memory")

    def close(self):
        if getattr(self, "_h", None):
            lib().or_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- operations --
    def append(self, seq, pos, tag, k, v) -> int:
        seq = np.ascontiguousarray(seq, dtype=np.int32)
        pos = np.ascontiguousarray(pos, dtype=np.int32)
        tag = np.ascontiguousarray(tag, dtype=np.uint8)
        k16, v16 = _u16(k), _u16(v)
        n = seq.shape[0]
        assert k16.size == n * self.H * self.d and v16.size == n * self.H * self.d
        return int(lib().or_append(self._h, n, _ptr(seq), _ptr(pos), _ptr(tag),
                                   _ptr(k16), _ptr(v16)))

    def evict(self, seq, budget, order: Optional[Sequence[int]] = None) -> int:
        seq = np.ascontiguousarray(seq, dtype=np.int32)
        budget = np.ascontiguousarray(budget, dtype=np.int32)
        o = None if order is None else np.ascontiguousarray(order, dtype=np.uint8)
        return int(lib().or_evict(self._h, seq.shape[0], _ptr(seq), _ptr(budget),
                                  None if o is None else _ptr(o)))

    def tbe(self, seq, pos, tag, t_min: int = 0, schedule: Optional[Sequence[int]] = None) -> int:
        """TBE after an append of the same tokens (see or_tbe)."""
        seq = np.ascontiguousarray(seq, dtype=np.int32)
        pos = np.ascontiguousarray(pos, dtype=np.int32)
        tag = np.ascontiguousarray(tag, dtype=np.uint8)
        sch = None if schedule is None else np.ascontiguousarray(schedule, dtype=np.int32)
        return int(lib().or_tbe(self._h, seq.shape[0], _ptr(seq), _ptr(pos), _ptr(tag),
                                int(t_min), None if sch is None else _ptr(sch)))

    def evict_slots(self, seq, cls, idx) -> int:
        """Explicit victims: (sequence, class, FIFO counter) each (see or_evict_slots)."""
        seq = np.ascontiguousarray(seq, dtype=np.int32)
        cls = np.ascontiguousarray(cls, dtype=np.uint8)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        return int(lib().or_evict_slots(self._h, seq.shape[0], _ptr(seq), _ptr(cls), _ptr(idx)))

    def compact_into(self, dst: "Oracle", seq) -> int:
        """Gather the live tokens of `seq` into the empty oracle `dst` (see or_compact)."""
        seq = np.ascontiguousarray(seq, dtype=np.int32)
        return int(lib().or_compact(self._h, dst._h, seq.shape[0], _ptr(seq)))

    def decode(self, seq, q, softmax_scale: float = 0.0, topk: Optional[int] = None,
               threads: int = 1):
        """fp64 attention output [n, Hq, d] and (if topk) top-k mass [n, Hq]."""
        seq = np.ascontiguousarray(seq, dtype=np.int32)
        q16 = _u16(q)
        n = seq.shape[0]
        assert q16.size == n * self.Hq * self.d
        out = np.zeros((n, self.Hq, self.d), dtype=np.float64)
        mass = np.zeros((n, self.Hq), dtype=np.float64) if topk else None
        st = lib().or_decode(self._h, n, _ptr(seq), _ptr(q16), float(softmax_scale),
                             int(topk or 0), _ptr(out), None if mass is None else _ptr(mass),
                             int(threads))
        if st != OK:
            raise ValueError(f"oracle decode rejected the call (status {st})")
        return out, mass

    # -- state export (copies) --
    def _arr(self, fn, dtype, shape, *args):
        p = getattr(lib(), fn)(self._h, *args)
        n = int(np.prod(shape))
        if n == 0:
            return np.zeros(shape, dtype=dtype)
        buf = (C.c_char * (n * np.dtype(dtype).itemsize)).from_address(p)
        return np.frombuffer(buf, dtype=dtype).reshape(shape).copy()

    def codes(self, c: int) -> np.ndarray:
        dt = np.uint16 if self.bits[c] == 16 else np.uint8
        return self._arr("or_codes", dt, (self.pool_pages[c], self.H, 2, PAGE, self.d), c)

    def params(self, c: int) -> Optional[np.ndarray]:
        if self.bits[c] == 16:
            return None
        return self._arr("or_params", np.uint16,
                         (self.pool_pages[c], self.H, 2, PAGE, self.d // self.G, 2), c)

    def slot_pos(self, c: int) -> np.ndarray:
        return self._arr("or_slot_pos", np.int32, (self.pool_pages[c], PAGE), c)

    def state(self) -> dict:
        ns, nb, cap = self.max_seqs, self.max_blocks, self.max_blocks * PAGE
        return {
            "table": self._arr("or_table", np.uint64, (ns, nb)),
            "num_blocks": self._arr("or_num_blocks", np.int32, (ns,)),
            "free_slots": self._arr("or_free_slots", np.int32, (ns, 3, cap)),
            "free_top": self._arr("or_free_top", np.int32, (ns, 3)),
            "fifo": self._arr("or_fifo", np.int32, (ns, 3, cap)),
            "fifo_head": self._arr("or_fifo_head", np.int32, (ns, 3)),
            "fifo_tail": self._arr("or_fifo_tail", np.int32, (ns, 3)),
            "live_count": self._arr("or_live_count", np.int32, (ns,)),
            "live_list": self._arr("or_live_list", np.uint64, (ns, nb)),
            "live_index": self._arr("or_live_index", np.int32, (ns, nb)),
            "num_live": self._arr("or_num_live", np.int32, (ns,)),
            "page_bump": self._arr("or_page_bump", np.int32, (3,)),
            "seg": self._arr("or_seg", np.int32, (ns, nb * PAGE, 5)),
            "nseg": self._arr("or_nseg", np.int32, (ns,)),
            "slot_pos": [self.slot_pos(c) for c in range(3)],
        }


def entry_page(e):
    return (np.asarray(e, dtype=np.uint64) & np.uint64(0xFFFFFFFF)).astype(np.int64)


def entry_class(e):
    return ((np.asarray(e, dtype=np.uint64) >> np.uint64(32)) & np.uint64(0xFF)).astype(np.int64)


def entry_mask(e):
    return ((np.asarray(e, dtype=np.uint64) >> np.uint64(48)) & np.uint64(0xFFFF)).astype(np.int64)


def live_entry(x):
    """Table entry index held in a live-list descriptor (page | class<<32 | entry<<40)."""
    return (np.asarray(x, dtype=np.uint64) >> np.uint64(40)).astype(np.int64)

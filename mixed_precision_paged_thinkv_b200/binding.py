"""ctypes binding of libthinkv.so (declared in include/thinkv.h).

Argument marshalling only: every step of append / evict / decode runs in the
library's CUDA kernels.  PyTorch provides the device memory (caller-owned
buffers and workspaces) and the stream.  There is no CPU fallback: if the
shared library is missing or cannot be loaded, importing ``lib()`` raises.
"""
from __future__ import annotations

import ctypes as C
import os
import threading
from typing import Optional, Sequence

import numpy as np
import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libthinkv.so")

OK, ERR_INVALID, ERR_OUT_OF_PAGES, ERR_OUT_OF_BLOCKS = 0, 1, 2, 3
ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = 4, 5, 6
R, E, T = 0, 1, 2
PAGE = 16

BUFFERS = ["pool_R", "pool_E", "pool_T", "slot_pos_R", "slot_pos_E", "slot_pos_T",
           "block_table", "num_blocks", "free_slots", "free_top", "fifo", "fifo_head",
           "fifo_tail", "live_count", "live_list", "live_index", "num_live", "page_bump",
           "status"]

EXPORTED = [
    "thinkv_layout_check", "thinkv_page_head_bytes", "thinkv_buffer_bytes",
    "thinkv_cache_reset", "thinkv_append_workspace_bytes", "thinkv_append_quantize",
    "thinkv_append_evict",
    "thinkv_evict", "thinkv_decode_workspace_bytes", "thinkv_decode_attention",
    "thinkv_get_status", "thinkv_clear_status", "thinkv_status_string",
    "thinkv_decode_attention_noalloc", "thinkv_classify_thoughts",
    "thinkv_tbe_buffer_bytes", "thinkv_tbe_reset", "thinkv_tbe_workspace_bytes", "thinkv_evict_tbe",
    "thinkv_evict_slots_workspace_bytes", "thinkv_evict_slots",
    "thinkv_compact_workspace_bytes", "thinkv_compact",
]

TBE_BUFFERS = ["seg", "nseg", "settled"]


class ThinkvError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})" if what else status_string(code))


class Layout(C.Structure):
    _fields_ = [("num_q_heads", C.c_int32), ("num_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("page_size", C.c_int32),
                ("group_size", C.c_int32), ("bits", C.c_int32 * 3),
                ("max_seqs", C.c_int32), ("max_blocks_per_seq", C.c_int32),
                ("pool_pages", C.c_int32 * 3), ("fmt", C.c_int32 * 3)]


class CacheStruct(C.Structure):
    _fields_ = [("L", Layout), ("pool", C.c_void_p * 3), ("slot_pos", C.c_void_p * 3),
                ("block_table", C.c_void_p), ("num_blocks", C.c_void_p),
                ("free_slots", C.c_void_p), ("free_top", C.c_void_p), ("fifo", C.c_void_p),
                ("fifo_head", C.c_void_p), ("fifo_tail", C.c_void_p),
                ("live_count", C.c_void_p), ("live_list", C.c_void_p),
                ("live_index", C.c_void_p), ("num_live", C.c_void_p),
                ("page_bump", C.c_void_p), ("status", C.c_void_p)]


class TbeStruct(C.Structure):
    _fields_ = [("seg", C.c_void_p), ("nseg", C.c_void_p), ("settled", C.c_void_p)]


_lock = threading.Lock()
_lib = None


def lib():
    """Load libthinkv.so (in-tree); raises if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"libthinkv.so not built ({LIB_PATH}); run "
                                  "`python -m mixed_precision_paged_thinkv_b200.build`")
            L = C.CDLL(LIB_PATH)
            P, I32, SZ = C.c_void_p, C.c_int32, C.c_size_t
            L.thinkv_layout_check.argtypes = [C.POINTER(Layout)]
            L.thinkv_layout_check.restype = C.c_int
            L.thinkv_page_head_bytes.argtypes = [C.POINTER(Layout), I32]
            L.thinkv_page_head_bytes.restype = SZ
            L.thinkv_buffer_bytes.argtypes = [C.POINTER(Layout), I32]
            L.thinkv_buffer_bytes.restype = SZ
            L.thinkv_cache_reset.argtypes = [C.POINTER(CacheStruct), P]
            L.thinkv_cache_reset.restype = C.c_int
            L.thinkv_append_workspace_bytes.argtypes = [C.POINTER(Layout), I32]
            L.thinkv_append_workspace_bytes.restype = SZ
            L.thinkv_append_quantize.argtypes = [C.POINTER(CacheStruct), I32, P, P, P, P, P, P, SZ, P]
            L.thinkv_append_quantize.restype = C.c_int
            L.thinkv_append_evict.argtypes = [C.POINTER(CacheStruct), I32, P, P, P, P, P, P, P, P, SZ, P]
            L.thinkv_append_evict.restype = C.c_int
            L.thinkv_evict.argtypes = [C.POINTER(CacheStruct), I32, P, P, P, P]
            L.thinkv_evict.restype = C.c_int
            L.thinkv_decode_workspace_bytes.argtypes = [C.POINTER(Layout), I32, I32]
            L.thinkv_decode_workspace_bytes.restype = SZ
            L.thinkv_decode_attention.argtypes = [C.POINTER(CacheStruct), I32, P, P, P, P, I32,
                                                  C.c_float, P, SZ, P]
            L.thinkv_decode_attention.restype = C.c_int
            L.thinkv_get_status.argtypes = [C.POINTER(CacheStruct), P, C.POINTER(I32)]
            L.thinkv_get_status.restype = C.c_int
            L.thinkv_clear_status.argtypes = [C.POINTER(CacheStruct), P]
            L.thinkv_clear_status.restype = C.c_int
            L.thinkv_classify_thoughts.argtypes = [I32, I32, P, C.c_float, C.c_float, P, P]
            L.thinkv_tbe_buffer_bytes.argtypes = [C.POINTER(Layout), I32]
            L.thinkv_tbe_buffer_bytes.restype = SZ
            L.thinkv_tbe_reset.argtypes = [C.POINTER(Layout), C.POINTER(TbeStruct), P]
            L.thinkv_tbe_reset.restype = C.c_int
            L.thinkv_evict_slots_workspace_bytes.argtypes = [I32]
            L.thinkv_evict_slots_workspace_bytes.restype = SZ
            L.thinkv_evict_slots.argtypes = [C.POINTER(CacheStruct), I32, P, P, P, P, SZ, P]
            L.thinkv_evict_slots.restype = C.c_int
            L.thinkv_tbe_workspace_bytes.argtypes = [I32]
            L.thinkv_tbe_workspace_bytes.restype = SZ
            L.thinkv_evict_tbe.argtypes = [C.POINTER(CacheStruct), C.POINTER(TbeStruct), I32, P, P, P,
                                           I32, P, P, SZ, P]
            L.thinkv_evict_tbe.restype = C.c_int
            L.thinkv_compact_workspace_bytes.argtypes = [I32, I32]
            L.thinkv_compact_workspace_bytes.restype = SZ
            L.thinkv_compact.argtypes = [C.POINTER(CacheStruct), C.POINTER(CacheStruct), I32, P, I32,
                                         P, SZ, P]
            L.thinkv_compact.restype = C.c_int
            L.thinkv_classify_thoughts.restype = C.c_int
            L.thinkv_status_string.argtypes = [I32]
            L.thinkv_status_string.restype = C.c_char_p
            _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().thinkv_status_string(int(code)).decode()


def classify_thoughts(mass: torch.Tensor, theta_t: float, theta_r: float,
                      tags: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """R/E/T tags (uint8 [n]) from top-k attention masses (fp32 [n, Hq], device)."""
    assert mass.dtype == torch.float32 and mass.dim() == 2 and mass.is_contiguous()
    n, hq = mass.shape
    if tags is None:
        tags = torch.empty(n, dtype=torch.uint8, device=mass.device)
    _check(lib().thinkv_classify_thoughts(int(n), int(hq), _ptr(mass), float(theta_t),
                                          float(theta_r), _ptr(tags), _stream(stream)),
           "classify_thoughts")
    return tags


def make_layout(num_q_heads, num_kv_heads, head_dim, group_size, bits, max_seqs,
                max_blocks_per_seq, pool_pages, fmt=(0, 0, 0)) -> Layout:
    return Layout(int(num_q_heads), int(num_kv_heads), int(head_dim), PAGE, int(group_size),
                  (C.c_int32 * 3)(*[int(b) for b in bits]), int(max_seqs),
                  int(max_blocks_per_seq), (C.c_int32 * 3)(*[int(p) for p in pool_pages]),
                  (C.c_int32 * 3)(*[int(f) for f in fmt]))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(code: int, what: str):
    if code != OK:
        raise ThinkvError(code, what)


class ThinKVCache:
    """One ThinKV cache (one attention layer) in device memory.

    Buffers are torch tensors owned by this object; the C ABI sees raw device
    pointers.  ``bits`` are the code widths of R, E, T (default 8/4/2).
    """

    def __init__(self, num_q_heads: int, num_kv_heads: int, head_dim: int, group_size: int,
                 bits: Sequence[int], max_seqs: int, max_blocks_per_seq: int,
                 pool_pages: Sequence[int], device: str = "cuda", tbe: bool = False,
                 fmt: Sequence[int] = (0, 0, 0)):
        self.layout = make_layout(num_q_heads, num_kv_heads, head_dim, group_size, bits,
                                  max_seqs, max_blocks_per_seq, pool_pages, fmt)
        self.fmt = tuple(int(f) for f in fmt)
        L = lib()
        _check(L.thinkv_layout_check(C.byref(self.layout)), "layout")
        self.Hq, self.H, self.d, self.G = num_q_heads, num_kv_heads, head_dim, group_size
        self.bits = tuple(int(b) for b in bits)
        self.max_seqs, self.max_blocks = int(max_seqs), int(max_blocks_per_seq)
        self.pool_pages = tuple(int(p) for p in pool_pages)
        self.device = torch.device(device)
        self.buf = {}
        for i, name in enumerate(BUFFERS):
            nbytes = int(L.thinkv_buffer_bytes(C.byref(self.layout), i))
            self.buf[name] = (torch.empty(nbytes, dtype=torch.uint8, device=self.device)
                              if nbytes > 0 else None)
        self.cs = CacheStruct()
        self.cs.L = self.layout
        for c, n in enumerate("RET"):
            self.cs.pool[c] = _ptr(self.buf[f"pool_{n}"])
            self.cs.slot_pos[c] = _ptr(self.buf[f"slot_pos_{n}"])
        for name in BUFFERS[6:]:
            setattr(self.cs, name, _ptr(self.buf[name]))
        self._ws = {}
        self.tbe = None
        if tbe:
            self.tbe_buf = {}
            for i, name in enumerate(TBE_BUFFERS):
                nbytes = int(L.thinkv_tbe_buffer_bytes(C.byref(self.layout), i))
                self.tbe_buf[name] = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            self.tbe = TbeStruct(*[_ptr(self.tbe_buf[n]) for n in TBE_BUFFERS])
        self.reset()

    # -- helpers --
    def page_head_bytes(self, c: int) -> int:
        return int(lib().thinkv_page_head_bytes(C.byref(self.layout), c))

    def _workspace(self, key: str, nbytes: int) -> torch.Tensor:
        # zero-filled once: the append and decode workspaces start with arrival
        # counters that every completed call leaves at zero
        t = self._ws.get(key)
        if t is None or t.numel() < nbytes:
            t = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
            self._ws[key] = t
        return t

    # -- operations --
    def reset(self, stream=None):
        _check(lib().thinkv_cache_reset(C.byref(self.cs), _stream(stream)), "reset")
        if self.tbe is not None:
            _check(lib().thinkv_tbe_reset(C.byref(self.layout), C.byref(self.tbe), _stream(stream)),
                   "tbe_reset")

    def evict_slots(self, seq: torch.Tensor, cls: torch.Tensor, fifo_index: torch.Tensor, stream=None):
        """Explicit victims: (sequence, class, FIFO counter) each, evicted in order."""
        n = int(seq.numel())
        if n == 0:
            return
        assert seq.dtype == torch.int32 and cls.dtype == torch.uint8 and fifo_index.dtype == torch.int32
        assert cls.numel() == n and fifo_index.numel() == n
        nbytes = int(lib().thinkv_evict_slots_workspace_bytes(n))
        ws = self._workspace("evict_slots", nbytes)
        _check(lib().thinkv_evict_slots(C.byref(self.cs), n, _ptr(seq), _ptr(cls), _ptr(fifo_index),
                                        _ptr(ws), ws.numel(), _stream(stream)), "evict_slots")

    def evict_tbe(self, seq: torch.Tensor, pos: torch.Tensor, tag: torch.Tensor, t_min: int = 0,
                  schedule: Optional[Sequence[int]] = None, stream=None):
        """TBE after an append of the same tokens (needs tbe=True)."""
        assert self.tbe is not None, "cache created without TBE buffers"
        n = int(seq.numel())
        assert seq.dtype == torch.int32 and pos.dtype == torch.int32 and tag.dtype == torch.uint8
        sch = None if schedule is None else (C.c_int32 * 3)(*[int(x) for x in schedule])
        nbytes = int(lib().thinkv_tbe_workspace_bytes(n))
        ws = self._workspace("tbe", nbytes)
        _check(lib().thinkv_evict_tbe(C.byref(self.cs), C.byref(self.tbe), n, _ptr(seq), _ptr(pos),
                                      _ptr(tag), int(t_min),
                                      None if sch is None else C.cast(sch, C.c_void_p),
                                      _ptr(ws), ws.numel(), _stream(stream)), "evict_tbe")

    def append(self, seq: torch.Tensor, pos: torch.Tensor, tag: torch.Tensor,
               k: torch.Tensor, v: torch.Tensor, stream=None):
        n = int(seq.numel())
        if n == 0:
            return
        assert seq.dtype == torch.int32 and pos.dtype == torch.int32 and tag.dtype == torch.uint8
        assert k.dtype == torch.float16 and v.dtype == torch.float16
        assert k.is_contiguous() and v.is_contiguous() and k.numel() == n * self.H * self.d
        nbytes = int(lib().thinkv_append_workspace_bytes(C.byref(self.layout), n))
        ws = self._workspace("append", nbytes)
        _check(lib().thinkv_append_quantize(C.byref(self.cs), n, _ptr(seq), _ptr(pos), _ptr(tag),
                                            _ptr(k), _ptr(v), _ptr(ws), ws.numel(),
                                            _stream(stream)), "append")

    def append_evict(self, seq: torch.Tensor, pos: torch.Tensor, tag: torch.Tensor,
                     k: torch.Tensor, v: torch.Tensor, budget: torch.Tensor,
                     order: Optional[Sequence[int]] = None, stream=None):
        """Append, then evict each sequence of the call to its budget (one launch
        for calls of up to 512 tokens).  budget: int32 per token; the value at
        each sequence's first token counts."""
        n = int(seq.numel())
        if n == 0:
            return
        assert seq.dtype == torch.int32 and pos.dtype == torch.int32 and tag.dtype == torch.uint8
        assert budget.dtype == torch.int32 and budget.numel() == n
        assert k.dtype == torch.float16 and v.dtype == torch.float16
        assert k.is_contiguous() and v.is_contiguous() and k.numel() == n * self.H * self.d
        nbytes = int(lib().thinkv_append_workspace_bytes(C.byref(self.layout), n))
        ws = self._workspace("append", nbytes)
        o = None if order is None else (C.c_uint8 * 3)(*order)
        _check(lib().thinkv_append_evict(C.byref(self.cs), n, _ptr(seq), _ptr(pos), _ptr(tag),
                                         _ptr(k), _ptr(v), _ptr(budget),
                                         None if o is None else C.cast(o, C.c_void_p),
                                         _ptr(ws), ws.numel(), _stream(stream)), "append_evict")

    def evict(self, seq: torch.Tensor, budget: torch.Tensor, order: Optional[Sequence[int]] = None,
              stream=None):
        n = int(seq.numel())
        assert seq.dtype == torch.int32 and budget.dtype == torch.int32
        o = None
        if order is not None:
            o = (C.c_uint8 * 3)(*[int(x) for x in order])
        _check(lib().thinkv_evict(C.byref(self.cs), n, _ptr(seq), _ptr(budget),
                                  None if o is None else C.cast(o, C.c_void_p),
                                  _stream(stream)), "evict")

    def compact_into(self, dst: "ThinKVCache", seq: torch.Tensor, max_tokens: int, stream=None):
        """Gather compaction of `seq`'s live tokens into the empty cache `dst`."""
        n = int(seq.numel())
        assert seq.dtype == torch.int32
        nbytes = int(lib().thinkv_compact_workspace_bytes(n, int(max_tokens)))
        ws = self._workspace("compact", nbytes)
        _check(lib().thinkv_compact(C.byref(self.cs), C.byref(dst.cs), n, _ptr(seq),
                                    int(max_tokens), _ptr(ws), ws.numel(), _stream(stream)),
               "compact")

    def decode_workspace_bytes(self, n: int, topk: int = 0) -> int:
        return int(lib().thinkv_decode_workspace_bytes(C.byref(self.layout), n, topk))

    def decode(self, seq: torch.Tensor, q: torch.Tensor, topk: Optional[int] = None,
               softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
               mass: Optional[torch.Tensor] = None, stream=None):
        n = int(seq.numel())
        assert seq.dtype == torch.int32 and q.dtype == torch.float16 and q.is_contiguous()
        if out is None:
            out = torch.empty(n, self.Hq, self.d, dtype=torch.float16, device=self.device)
        if topk and mass is None:
            mass = torch.empty(n, self.Hq, dtype=torch.float32, device=self.device)
        nbytes = self.decode_workspace_bytes(n, int(topk or 0))
        if nbytes == 0:
            raise ThinkvError(ERR_INVALID, "decode workspace size")
        ws = self._workspace("decode", nbytes)
        _check(lib().thinkv_decode_attention(C.byref(self.cs), n, _ptr(seq), _ptr(q), _ptr(out),
                                             _ptr(mass) if topk else None, int(topk or 0),
                                             float(softmax_scale), _ptr(ws), ws.numel(),
                                             _stream(stream)), "decode")
        return out, (mass if topk else None)

    def status(self, stream=None) -> int:
        v = C.c_int32(0)
        _check(lib().thinkv_get_status(C.byref(self.cs), _stream(stream), C.byref(v)), "status")
        return int(v.value)

    def clear_status(self, stream=None):
        _check(lib().thinkv_clear_status(C.byref(self.cs), _stream(stream)), "clear_status")

    # -- state snapshot (host copies, for comparisons and checkpoints) --
    def _host(self, name, dtype, shape):
        t = self.buf[name]
        if t is None:
            return np.zeros(shape, dtype=dtype)
        return t.cpu().numpy().view(dtype).reshape(shape).copy()

    def snapshot(self) -> dict:
        ns, nb = self.max_seqs, self.max_blocks
        cap = nb * PAGE
        st = {
            "table": self._host("block_table", np.uint64, (ns, nb)),
            "num_blocks": self._host("num_blocks", np.int32, (ns,)),
            "free_slots": self._host("free_slots", np.int32, (ns, 3, cap)),
            "free_top": self._host("free_top", np.int32, (ns, 3)),
            "fifo": self._host("fifo", np.int32, (ns, 3, cap)),
            "fifo_head": self._host("fifo_head", np.int32, (ns, 3)),
            "fifo_tail": self._host("fifo_tail", np.int32, (ns, 3)),
            "live_count": self._host("live_count", np.int32, (ns,)),
            "live_list": self._host("live_list", np.uint64, (ns, nb)),
            "live_index": self._host("live_index", np.int32, (ns, nb)),
            "num_live": self._host("num_live", np.int32, (ns,)),
            "page_bump": self._host("page_bump", np.int32, (3,)),
            "slot_pos": [self._host(f"slot_pos_{n}", np.int32, (self.pool_pages[c], PAGE))
                         for c, n in enumerate("RET")],
        }
        if self.tbe is not None:
            seg = self.tbe_buf["seg"].cpu().numpy().view(np.int32).reshape(ns, cap, 4)
            # (class | level << 8, lo, len, trim) -> (class, level, lo, len, trim)
            st["seg"] = np.stack([seg[..., 0] & 0xFF, (seg[..., 0] >> 8) & 0xFF, seg[..., 1],
                                  seg[..., 2], seg[..., 3]], axis=-1)
            st["nseg"] = self.tbe_buf["nseg"].cpu().numpy().view(np.int32).copy()
        return st

    def pool_bytes(self, c: int) -> np.ndarray:
        """Raw bytes of class c's pool: [pool_pages][Hkv][page_head_bytes]."""
        n = "RET"[c]
        return self._host(f"pool_{n}", np.uint8,
                          (self.pool_pages[c], self.H, self.page_head_bytes(c)))

"""The C ABI library loads, exports every entry point include/thinkv.h
declares, and its host-only functions behave (no GPU needed)."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from mixed_precision_paged_thinkv_b200 import build, binding
    build.build()
    return binding.lib()


def _declared():
    hdr = open(os.path.join(ROOT, "include", "thinkv.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(thinkv_[a-z_]+)\s*\(", hdr)))


def test_every_declared_symbol_is_exported(lib):
    from mixed_precision_paged_thinkv_b200 import binding
    declared = _declared()
    assert declared, "no declarations found"
    assert set(declared) == set(binding.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (thinkv_\w+)", out))
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    # nothing else leaks out of the library under the thinkv_ prefix
    assert exported == set(declared)


def _layout(**kw):
    from mixed_precision_paged_thinkv_b200 import binding
    a = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, group_size=64, bits=(8, 4, 2),
             max_seqs=16, max_blocks_per_seq=100, pool_pages=(10, 20, 30))
    a.update(kw)
    return binding.make_layout(**a)


def test_layout_check_and_sizes(lib):
    L = _layout()
    assert lib.thinkv_layout_check(C.byref(L)) == 0
    d, G = 128, 64
    for c, b in enumerate((8, 4, 2)):
        assert lib.thinkv_page_head_bytes(C.byref(L), c) == 4 * d * b + 128 * (d // G)
    assert lib.thinkv_page_head_bytes(C.byref(L), 0) == 4352
    assert lib.thinkv_buffer_bytes(C.byref(L), 0) == 10 * 8 * 4352
    assert lib.thinkv_buffer_bytes(C.byref(L), 6) == 16 * 100 * 8      # block table
    assert lib.thinkv_buffer_bytes(C.byref(L), 8) == 16 * 3 * 1600 * 4  # free slots
    assert lib.thinkv_buffer_bytes(C.byref(L), 18) == 4
    assert lib.thinkv_buffer_bytes(C.byref(L), 19) == 0
    L16 = _layout(bits=(16, 16, 16))
    assert lib.thinkv_page_head_bytes(C.byref(L16), 2) == 64 * d
    for bad in (dict(head_dim=96), dict(group_size=16), dict(bits=(8, 3, 2)),
                dict(num_q_heads=36), dict(num_q_heads=72, num_kv_heads=8),
                dict(max_seqs=0), dict(max_seqs=70000), dict(pool_pages=(-1, 0, 0))):
        Lb = _layout(**bad)
        assert lib.thinkv_layout_check(C.byref(Lb)) == 1, bad
        assert lib.thinkv_buffer_bytes(C.byref(Lb), 0) == 0


def test_host_validation_without_launch(lib):
    """Bad arguments are rejected before anything reaches the GPU."""
    from mixed_precision_paged_thinkv_b200 import binding
    cs = binding.CacheStruct()
    cs.L = _layout()
    # null buffers -> invalid, no CUDA call made
    assert lib.thinkv_cache_reset(C.byref(cs), None) == 1
    assert lib.thinkv_append_quantize(C.byref(cs), 4, None, None, None, None, None, None, 0, None) == 1
    assert lib.thinkv_evict(C.byref(cs), 1, None, None, None, None) == 1
    assert lib.thinkv_decode_attention(C.byref(cs), 1, None, None, None, None, 0, 0.0, None, 0, None) == 1
    # a cache struct whose pointers are non-null but bad sizes/orders
    fake = C.c_void_p(16)
    for name, _ in binding.CacheStruct._fields_[1:]:
        v = getattr(cs, name)
        if isinstance(v, C.Array):
            for i in range(3):
                v[i] = 16
        else:
            setattr(cs, name, 16)
    assert lib.thinkv_append_quantize(C.byref(cs), -1, fake, fake, fake, fake, fake, fake, 10 ** 6, None) == 1
    assert lib.thinkv_append_quantize(C.byref(cs), 0, None, None, None, None, None, None, 0, None) == 0
    assert lib.thinkv_append_quantize(C.byref(cs), 8, fake, fake, fake, fake, fake, fake, 8, None) == 6
    bad_order = (C.c_uint8 * 3)(2, 2, 0)
    assert lib.thinkv_evict(C.byref(cs), 1, fake, fake, C.cast(bad_order, C.c_void_p), None) == 1
    assert lib.thinkv_evict(C.byref(cs), 0, None, None, None, None) == 0
    assert lib.thinkv_decode_attention(C.byref(cs), 0, fake, fake, fake, None, 0, 0.0, fake, 1, None) == 1
    assert lib.thinkv_decode_attention(C.byref(cs), 1, fake, fake, fake, fake, 65, 0.0, fake, 1, None) == 1
    assert lib.thinkv_append_workspace_bytes(C.byref(cs.L), 1000) >= 1000 * 4


def test_status_strings(lib):
    for code in range(7):
        assert lib.thinkv_status_string(code)
    assert lib.thinkv_status_string(99) == b"unknown status"


def test_layout_decoder_is_a_bijection():
    """The test-side layout decoder maps every (slot, channel) to its own bits."""
    from layout_decode import _maps
    for d, G in ((64, 32), (128, 64), (128, 32), (64, 64)):
        for b in (2, 4, 8, 16):
            kb, ks, vb, vs = _maps(d, G, b)
            w = 16 if b == 16 else b
            for bo, sh, lo in ((kb, ks, 0), (vb, vs, 2 * d * b if b < 16 else 32 * d)):
                bits = (bo - lo) * 8 + sh
                assert bits.min() == 0 and bits.max() == 16 * d * w - w
                assert len(np.unique(bits)) == 16 * d
                assert np.all(bits % w == 0)


def test_misaligned_pointers_rejected_without_launch(lib):
    """Pointers off the documented boundaries are refused before any CUDA call
    (bulk copies and vector accesses would otherwise fault on the device)."""
    from mixed_precision_paged_thinkv_b200 import binding
    cs = binding.CacheStruct()
    cs.L = _layout()
    for name, _ in binding.CacheStruct._fields_[1:]:
        v = getattr(cs, name)
        if isinstance(v, C.Array):
            for i in range(3):
                v[i] = 4096
        else:
            setattr(cs, name, 4096)
    ok = C.c_void_p(4096)
    odd = C.c_void_p(4096 + 2)
    word = C.c_void_p(4096 + 4)       # 4-byte aligned, not 16
    # a misaligned k, v, q, out or workspace
    assert lib.thinkv_append_quantize(C.byref(cs), 4, ok, ok, ok, word, ok, ok, 10 ** 6, None) == 1
    assert lib.thinkv_append_quantize(C.byref(cs), 4, ok, ok, ok, ok, word, ok, 10 ** 6, None) == 1
    assert lib.thinkv_append_quantize(C.byref(cs), 4, odd, ok, ok, ok, ok, ok, 10 ** 6, None) == 1
    assert lib.thinkv_append_quantize(C.byref(cs), 4, ok, ok, ok, ok, ok, word, 10 ** 6, None) == 1
    assert lib.thinkv_evict(C.byref(cs), 1, odd, ok, None, None) == 1
    assert lib.thinkv_evict(C.byref(cs), 1, ok, odd, None, None) == 1
    assert lib.thinkv_decode_attention(C.byref(cs), 1, ok, word, ok, None, 0, 0.0, ok, 10 ** 6, None) == 1
    assert lib.thinkv_decode_attention(C.byref(cs), 1, ok, ok, word, None, 0, 0.0, ok, 10 ** 6, None) == 1
    assert lib.thinkv_decode_attention(C.byref(cs), 1, odd, ok, ok, None, 0, 0.0, ok, 10 ** 6, None) == 1
    assert lib.thinkv_decode_attention(C.byref(cs), 1, ok, ok, ok, odd, 8, 0.0, ok, 10 ** 6, None) == 1
    assert lib.thinkv_decode_attention(C.byref(cs), 1, ok, ok, ok, None, 0, 0.0, word, 10 ** 6, None) == 1
    f = lib.thinkv_decode_attention_noalloc
    f.argtypes = [C.POINTER(binding.CacheStruct), C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p,
                  C.c_void_p, C.c_int32, C.c_float, C.c_void_p]
    f.restype = C.c_int
    assert f(C.byref(cs), 1, ok, word, ok, None, 0, 0.0, None) == 1
    # a misaligned cache buffer makes every operation refuse the cache
    cs.pool[1] = 4096 + 8
    assert lib.thinkv_cache_reset(C.byref(cs), None) == 1
    assert lib.thinkv_evict(C.byref(cs), 1, ok, ok, None, None) == 1
    cs.pool[1] = 4096
    cs.block_table = 4096 + 4
    assert lib.thinkv_cache_reset(C.byref(cs), None) == 1
    cs.block_table = 4096
    cs.num_live = 4096 + 2
    assert lib.thinkv_cache_reset(C.byref(cs), None) == 1


def test_classify_host_validation(lib):
    ok = C.c_void_p(4096)
    f = lib.thinkv_classify_thoughts
    assert f(-1, 4, ok, C.c_float(0.5), C.c_float(0.2), ok, None) == 1
    assert f(4, 0, ok, C.c_float(0.5), C.c_float(0.2), ok, None) == 1
    assert f(4, 4, ok, C.c_float(float("nan")), C.c_float(0.2), ok, None) == 1
    assert f(4, 4, None, C.c_float(0.5), C.c_float(0.2), ok, None) == 1
    assert f(4, 4, C.c_void_p(4098), C.c_float(0.5), C.c_float(0.2), ok, None) == 1
    assert f(0, 4, None, C.c_float(0.5), C.c_float(0.2), None, None) == 0


def test_evict_slots_host_validation(lib):
    """thinkv_evict_slots refuses bad counts, missing or misaligned arrays and a
    short workspace before any CUDA call; zero victims is a no-op."""
    from mixed_precision_paged_thinkv_b200 import binding
    cs = binding.CacheStruct()
    cs.L = _layout()
    for name, _ in binding.CacheStruct._fields_[1:]:
        v = getattr(cs, name)
        if isinstance(v, C.Array):
            for i in range(3):
                v[i] = 4096
        else:
            setattr(cs, name, 4096)
    ok, odd = C.c_void_p(4096), C.c_void_p(4096 + 2)
    f = lib.thinkv_evict_slots
    need = lib.thinkv_evict_slots_workspace_bytes(8)
    assert need >= 8 * 4 and lib.thinkv_evict_slots_workspace_bytes(-1) == 0
    assert f(C.byref(cs), -1, ok, ok, ok, ok, need, None) == 1
    assert f(C.byref(cs), 8, None, ok, ok, ok, need, None) == 1
    assert f(C.byref(cs), 8, ok, None, ok, ok, need, None) == 1
    assert f(C.byref(cs), 8, ok, ok, None, ok, need, None) == 1
    assert f(C.byref(cs), 8, odd, ok, ok, ok, need, None) == 1        # seq not 4-byte aligned
    assert f(C.byref(cs), 8, ok, ok, odd, ok, need, None) == 1        # fifo_index likewise
    assert f(C.byref(cs), 8, ok, ok, ok, C.c_void_p(4096 + 4), need, None) == 1   # workspace
    assert f(C.byref(cs), 8, ok, ok, ok, ok, need - 1, None) == binding.ERR_WORKSPACE
    assert f(C.byref(cs), 8, ok, ok, ok, None, need, None) == binding.ERR_WORKSPACE
    assert f(C.byref(cs), 0, None, None, None, None, 0, None) == 0


def test_append_evict_host_validation(lib):
    """thinkv_append_evict refuses a missing or misaligned budget, a bad class
    order and the append's own bad arguments before any CUDA call."""
    from mixed_precision_paged_thinkv_b200 import binding
    cs = binding.CacheStruct()
    cs.L = _layout()
    for name, _ in binding.CacheStruct._fields_[1:]:
        v = getattr(cs, name)
        if isinstance(v, C.Array):
            for i in range(3):
                v[i] = 4096
        else:
            setattr(cs, name, 4096)
    ok, odd, word = C.c_void_p(4096), C.c_void_p(4096 + 2), C.c_void_p(4096 + 4)
    f = lib.thinkv_append_evict
    big = 10 ** 6
    bad_order = (C.c_uint8 * 3)(2, 2, 0)
    far_order = (C.c_uint8 * 3)(0, 1, 3)
    assert f(C.byref(cs), -1, ok, ok, ok, ok, ok, ok, None, ok, big, None) == 1
    assert f(C.byref(cs), 4, ok, ok, ok, ok, ok, None, None, ok, big, None) == 1       # no budget
    assert f(C.byref(cs), 4, ok, ok, ok, ok, ok, odd, None, ok, big, None) == 1        # budget misaligned
    assert f(C.byref(cs), 4, ok, ok, ok, word, ok, ok, None, ok, big, None) == 1       # k misaligned
    assert f(C.byref(cs), 4, ok, ok, ok, ok, ok, ok, C.cast(bad_order, C.c_void_p), ok, big, None) == 1
    assert f(C.byref(cs), 4, ok, ok, ok, ok, ok, ok, C.cast(far_order, C.c_void_p), ok, big, None) == 1
    assert f(C.byref(cs), 4, ok, ok, ok, ok, ok, ok, None, ok, 0, None) == binding.ERR_WORKSPACE
    assert f(C.byref(cs), 0, None, None, None, None, None, None, None, None, 0, None) == 0

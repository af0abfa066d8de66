"""thinkv_decode_attention_noalloc: decode for callers that cannot allocate
device memory where they decode (a host framework that owns all device memory
and gives its plugins no allocator, or paths that cannot pay for cudaMalloc's
device-wide synchronisation).  Its scratch is the library's fixed device array,
so its results must match the workspace entry point's, call after call.

This file is collected last on purpose: it must pass when run alone in a fresh
process (the first call on the device looks up the array's address) and after
every other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = 2e-3  # row-normalised max difference, the decode tolerance of the parity tests


def _rel(a, b):
    a = a.float().cpu().numpy().astype(np.float64).reshape(-1, a.shape[-1])
    b = b.float().cpu().numpy().astype(np.float64).reshape(-1, b.shape[-1])
    den = np.abs(b).max(axis=1)
    num = np.abs(a - b).max(axis=1)
    return float(np.where(den > 0, num / np.where(den > 0, den, 1), num).max())


def _noalloc(cache, seqs, q, out, mass, topk):
    from mixed_precision_paged_thinkv_b200 import binding
    lib = binding.lib()
    f = lib.thinkv_decode_attention_noalloc
    f.argtypes = [C.POINTER(binding.CacheStruct), C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p,
                  C.c_void_p, C.c_int32, C.c_float, C.c_void_p]
    f.restype = C.c_int
    return f(C.byref(cache.cs), int(seqs.numel()), seqs.data_ptr(), q.data_ptr(), out.data_ptr(),
             mass.data_ptr() if mass is not None else None, int(topk or 0), 0.0,
             torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name,topk", [("r1-llama-8b", None), ("gpt-oss-20b", 32)])
def test_noalloc_matches_workspace_decode_on_two_calls(name, topk):
    from mixed_precision_paged_thinkv_b200 import build, workloads as W
    from mixed_precision_paged_thinkv_b200.runner import WorkloadRun
    build.build()
    base = W.WORKLOADS[name]
    w = W.scaled(base, batch=5, lengths=("uniform", 900, 2600), churn_steps=0)
    run = WorkloadRun(w, extra=4)
    run.setup()
    seqs = run.all_seqs
    for step in range(2):
        q = W.q_values(w, step, device="cuda")
        ref, ref_mass = run.cache.decode(seqs, q, topk=topk)
        # two no-alloc calls in a row: the second finds the first one's leftovers
        for _ in range(2):
            out = torch.full_like(ref, float("nan"))
            mass = torch.full((w.batch, w.num_q_heads), float("nan"), device="cuda") if topk else None
            assert _noalloc(run.cache, seqs, q, out, mass, topk) == 0
            torch.cuda.synchronize()
            assert run.cache.status() == 0
            assert _rel(out, ref) <= TOL
            if topk:
                assert float((mass - ref_mass).abs().max()) <= TOL
        # one more step changes the cache before the next pair of calls
        run.churn_step()


def test_noalloc_rejects_calls_beyond_its_scratch():
    """A call whose scratch need exceeds the fixed array is refused before
    anything is launched (q and out are never touched, so small buffers do)."""
    from mixed_precision_paged_thinkv_b200 import binding, build
    build.build()
    n = 16384
    cache = binding.ThinKVCache(2048, 256, 128, 64, (8, 4, 2), n, 1, (1, 1, 1))
    seqs = torch.arange(n, dtype=torch.int32, device="cuda")
    q = torch.zeros(16, 128, dtype=torch.float16, device="cuda")
    out = torch.zeros_like(q)
    need = cache.decode_workspace_bytes(n, 0)
    assert need > binding_scratch_bytes()
    assert _noalloc(cache, seqs, q, out, None, None) == binding.ERR_WORKSPACE


def binding_scratch_bytes():
    import re
    import os
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "include", "thinkv.h")).read()
    m = re.search(r"#define THINKV_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", hdr)
    return int(m.group(1)) << int(m.group(2))

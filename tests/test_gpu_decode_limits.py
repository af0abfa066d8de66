"""Decode at the largest call the interface accepts (16,384 sequences in one
call), for both head dims, with and without the top-k statistic: the launch
plan (the per-CTA prefix of live pages, the page ring, the top-k buffers) fits
in shared memory, the call succeeds, and sequences with no live tokens give
zero rows and zero masses (the documented results for an empty sequence)."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,G,Hq,Hkv,topk", [
    (64, 32, 64, 8, 32),      # gpt-oss-20b's head shape, top-k 32
    (64, 32, 64, 8, None),
    (128, 64, 64, 8, 64),     # d = 128, eight query heads per kv-head, the largest k
])
def test_decode_at_the_largest_sequence_count(d, G, Hq, Hkv, topk):
    from mixed_precision_paged_thinkv_b200 import build
    from mixed_precision_paged_thinkv_b200.binding import ThinKVCache
    build.build()
    n = 16384
    cache = ThinKVCache(Hq, Hkv, d, G, (8, 4, 2), n, 1, (1, 1, 1))
    assert cache.decode_workspace_bytes(n, topk or 0) > 0
    seqs = torch.arange(n, dtype=torch.int32, device="cuda")
    q = torch.randn(n, Hq, d, device="cuda").half()
    out, mass = cache.decode(seqs, q, topk=topk)
    torch.cuda.synchronize()
    assert cache.status() == 0
    assert bool((out == 0).all())
    if topk:
        assert bool((mass == 0).all())

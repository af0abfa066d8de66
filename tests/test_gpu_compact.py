"""GPU parity of the gather-compaction baseline (thinkv_compact): the
compacted cache bit for bit against the oracle's compaction (tables, stacks,
FIFOs, live lists, slot positions, the codes and params of every live slot),
and decode over it within 2e-3 of the oracle."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from mixed_precision_paged_thinkv_b200 import workloads as W

import harness as Hn

pytestmark = pytest.mark.gpu


def _dev(a, dt):
    return torch.as_tensor(np.ascontiguousarray(a)).to("cuda", dt)


@pytest.mark.parametrize("seed", range(4))
def test_compaction_matches_oracle(seed):
    from mixed_precision_paged_thinkv_b200.binding import ThinKVCache
    rng = np.random.default_rng(seed)
    # every (head_dim, group_size) instantiation of the gather: (64|128) x (32|64)
    ns, L, H, d, G = 5, 700, 2, [64, 128][seed % 2], [32, 64][seed // 2]
    bits = [(8, 4, 2), (16, 4, 2), (2, 8, 16), (4, 4, 8)][seed]
    nb = L // 16 * 3 + 8
    pool = (ns * L // 16 + 8,) * 3
    args = (8, H, d, G, bits, ns, nb, pool)
    g, gd = ThinKVCache(*args, tbe=True), ThinKVCache(*args)
    o, od = O.Oracle(*args), O.Oracle(*args)
    for p0 in range(0, L, 140):
        seq = np.repeat(np.arange(ns, dtype=np.int32), 140)
        pos = np.tile(np.arange(p0, p0 + 140, dtype=np.int32), ns)
        tag = np.repeat(rng.integers(0, 3, ns * 140 // 7), 7).astype(np.uint8)
        kv = rng.standard_normal((2, len(seq), H, d)).astype(np.float16)
        k, v = torch.as_tensor(kv[0]), torch.as_tensor(kv[1])
        g.append(_dev(seq, torch.int32), _dev(pos, torch.int32), _dev(tag, torch.uint8), k.cuda(), v.cuda())
        g.evict_tbe(_dev(seq, torch.int32), _dev(pos, torch.int32), _dev(tag, torch.uint8),
                    t_min=4, schedule=[24, 12, 6])
        assert o.append(seq, pos, tag, k, v) == O.OK
        assert o.tbe(seq, pos, tag, t_min=4, schedule=[24, 12, 6]) == O.OK
        b = rng.integers(40, 400, ns).astype(np.int32)
        g.evict(_dev(np.arange(ns), torch.int32), _dev(b, torch.int32))
        assert o.evict(np.arange(ns, dtype=np.int32), b) == O.OK
    order = rng.permutation(ns).astype(np.int32)
    g.compact_into(gd, _dev(order, torch.int32), max_tokens=ns * L)
    assert o.compact_into(od, order) == O.OK
    torch.cuda.synchronize()
    assert g.status() == 0 and gd.status() == 0
    gs, os_ = gd.snapshot(), od.state()
    Hn.compare_state(gs, os_, ns)
    Hn.compare_codes(gd, od, os_, ns)
    Hn.check_slot_invariants(gs, ns)
    q = torch.as_tensor(rng.standard_normal((ns, 8, d)).astype(np.float16))
    out, mass = gd.decode(torch.arange(ns, dtype=torch.int32, device="cuda"), q.cuda(), topk=5)
    ref, rmass = od.decode(np.arange(ns, dtype=np.int32), q, topk=5, threads=8)
    err = Hn.attn_error(out.cpu().numpy(), ref)
    merr = float(np.abs(mass.cpu().numpy().astype(np.float64) - rmass).max())
    print(f"compaction seed {seed}: attention error {err:.3e}, mass error {merr:.3e}")
    assert err <= Hn.TOL and merr <= Hn.MASS_TOL


def test_compaction_of_a_reduced_churn_state_and_refusals():
    from mixed_precision_paged_thinkv_b200.binding import ThinKVCache, ThinkvError
    from mixed_precision_paged_thinkv_b200.runner import WorkloadRun
    w = W.scaled(W.WORKLOADS["churn"], batch=8, lengths=("loguniform", 300, 3000), churn_steps=30)
    run = WorkloadRun(w)
    run.setup()
    orun = Hn.OracleRun(w, run.geom)
    orun.setup()
    c = run.cache
    dst = ThinKVCache(w.num_q_heads, w.num_kv_heads, w.head_dim, w.group_size, w.bits,
                      c.max_seqs, c.max_blocks, c.pool_pages)
    od = O.Oracle(w.num_q_heads, w.num_kv_heads, w.head_dim, w.group_size, w.bits,
                  c.max_seqs, c.max_blocks, c.pool_pages)
    seqs = np.arange(w.batch, dtype=np.int32)
    # a bound below the live count is refused on the device (status), nothing changes
    c.compact_into(dst, _dev(seqs, torch.int32), max_tokens=10)
    torch.cuda.synchronize()
    assert dst.status() == 1
    dst.reset()
    c.compact_into(dst, _dev(seqs, torch.int32), max_tokens=10 ** 6)
    assert orun.o.compact_into(od, seqs) == O.OK
    torch.cuda.synchronize()
    assert dst.status() == 0
    Hn.compare_state(dst.snapshot(), od.state(), w.batch)
    Hn.compare_codes(dst, od, od.state(), w.batch)
    # a second compaction into the same sequences is refused (dst not empty)
    c.compact_into(dst, _dev(seqs[:1], torch.int32), max_tokens=10 ** 6)
    torch.cuda.synchronize()
    assert dst.status() == 1

"""GPU parity at the full workload sizes, in the launch configuration bench.py
times (every sequence of the batch decoded in one call).

Sequences are independent except for the global numbering of pages, so the
oracle replays a sample of sequences (the first, the middle, the last and the
longest) from the same generator and its results must equal the GPU's for
those sequences: the live set by position and class, the codes and params of
every live token (bit for bit), and the decode output rows (2e-3) and top-k
masses (2e-3).  The churn workload runs its 1000 steps (append one token per
sequence, evict to 5%, decode) with the slot invariants of every sequence and
the sampled oracle outputs checked every 100 steps.
"""
import numpy as np
import pytest
import torch

from mixed_precision_paged_thinkv_b200 import workloads as W

import harness as Hn

pytestmark = pytest.mark.gpu


def _sample(w, lengths):
    picks = [0, w.batch // 2, w.batch - 1, int(np.argmax(lengths))]
    return sorted(set(picks))


def _check(g, osub, step, topk):
    torch.cuda.synchronize()
    assert g.cache.status() == 0
    snap = g.cache.snapshot()
    Hn.check_slot_invariants(snap, g.w.batch)
    ost = osub.o.state()
    for j, s in enumerate(osub.seqs):
        Hn.compare_seq_structure(snap, s, ost, j)
        gl = Hn.gpu_live_by_pos(snap, s)
        ol = osub.live_by_pos(j)
        assert sorted(gl) == sorted(ol), f"live positions of seq {s}"
        assert all(gl[p][0] == ol[p][0] for p in gl), f"classes of seq {s}"
        Hn.compare_codes_by_pos(g.cache, gl, osub.o, ol)
    out, mass = g.decode(step, topk=topk)
    ref, rmass = osub.decode(step, topk=topk)
    got = out.cpu().numpy()[osub.seqs]
    err = Hn.attn_error(got, ref)
    print(f"{g.w.name} step {step}: attention error {err:.3e}")
    assert err <= Hn.TOL, err
    if topk:
        merr = float(np.abs(mass.cpu().numpy()[osub.seqs].astype(np.float64) - rmass).max())
        assert merr <= Hn.MASS_TOL, merr


# the '-mixed' cases keep the whole history live (R/E/T mix, 4- and 2-bit
# pages at full scale); the budgeted ones retain almost only R tokens
@pytest.mark.parametrize("name", ["r1-llama-8b", "r1-qwen-14b", "gpt-oss-20b",
                                  "r1-llama-8b-mixed", "gpt-oss-20b-mixed"])
def test_full_size_workloads(name):
    from mixed_precision_paged_thinkv_b200.runner import WorkloadRun
    w = W.get(name)
    g = WorkloadRun(w, extra=2)
    g.setup()
    osub = Hn.OracleSubset(w, _sample(w, g.sched.lengths), extra=2)
    osub.setup()
    _check(g, osub, 0, w.topk)
    g.churn_step()
    osub.churn_step()
    _check(g, osub, 1, w.topk)


def test_churn_1000_steps():
    from mixed_precision_paged_thinkv_b200.runner import WorkloadRun
    w = W.WORKLOADS["churn"]
    g = WorkloadRun(w, extra=0)
    # setup without the churn steps: they are the test
    for call in g.sched.prefill_calls():
        g.append_call(call)
    g.evict_all()
    osub = Hn.OracleSubset(w, _sample(w, g.sched.lengths), extra=0)
    osub.setup(churn=False)
    _check(g, osub, 0, w.topk)
    for step in range(1, w.churn_steps + 1):
        g.churn_step(decode=True, step=step)
        osub.churn_step()
        if step % w.check_every == 0:
            _check(g, osub, step, w.topk)

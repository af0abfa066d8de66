"""Host-side logic of bench.py: clock parsing, aggregation over replicas, and
the max/sum reduction over ranks (world size 2, gloo, CPU)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench

CSV = """index, clocks.sm [MHz], clocks.max.sm [MHz], power.draw [W], clocks_event_reasons.active, clocks_event_reasons.hw_slowdown, clocks_event_reasons.hw_thermal_slowdown, clocks_event_reasons.sw_thermal_slowdown, clocks_event_reasons.sw_power_cap
0, 1965 MHz, 1965 MHz, 400.1 W, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active
0, 1950 MHz, 1965 MHz, 700.3 W, 0x0000000000000004, Not Active, Not Active, Not Active, Active
0, 1900 MHz, 1965 MHz, 800.0 W, 0x0000000000000004, Not Active, Not Active, Not Active, Active
1, 1000 MHz, 1965 MHz, 100.0 W, 0x0000000000000008, Active, Not Active, Not Active, Not Active
"""


def test_parse_clocks_selects_gpu_and_reasons():
    c = bench.parse_clocks(CSV, index=0)
    assert c["sm_mhz"] == 1950.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"] and c["samples"] == 3
    c1 = bench.parse_clocks(CSV, index=1)
    assert c1["reasons"] == ["hw_slowdown"]
    assert bench.parse_clocks("")["sm_mhz"] is None


def test_aggregate_is_total_tokens_over_slowest_rank():
    v, worst = bench.aggregate([(160, 1.0), (160, 2.0)])
    assert worst == 2.0 and v == 160.0


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE="2", LOCAL_RANK=str(rank), THINKV_BENCH_BACKEND="gloo")
    world, r, _ = bench.dist_init()
    secs = [1.5, 2.5][r]
    toks = [16.0, 16.0][r]
    m, n = bench.dist_max_sum(secs, toks, world, torch.device("cpu"))
    bench.barrier(world)
    q.put((r, m, n))
    dist.destroy_process_group()


def test_replicas_reduce_max_time_and_sum_tokens_over_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for r, m, n in got:
        assert m == 2.5 and n == 32.0


def test_launches_per_step_counts_the_one_launch_append_path():
    import bench
    assert bench.launches_per_step(16) == 3
    assert bench.launches_per_step(512) == 3
    assert bench.launches_per_step(513) == 5


def test_before_eviction_workloads_keep_the_shape_and_history():
    """The supplementary '-mixed' workloads are the same layer and history with
    nothing evicted: same lengths and tags, budget = every generated token."""
    import numpy as np
    from mixed_precision_paged_thinkv_b200 import workloads as W
    for name, base in W.WORKLOADS.items():
        if name == "tiny":
            continue
        m = W.get(name + "-mixed")
        assert m.budget == ("frac", 1.0) and m.churn_steps == 0
        for f in ("batch", "num_q_heads", "num_kv_heads", "head_dim", "group_size", "bits",
                  "lengths", "segments", "tag_probs", "topk", "seed"):
            assert getattr(m, f) == getattr(base, f), (name, f)
        sb, sm = W.Schedule(base, 0), W.Schedule(m, 0)
        assert np.array_equal(sb.lengths, sm.lengths)
        n = int(sb.lengths[0])                      # the history (churn steps extend the base)
        assert np.array_equal(sb.tags(0)[:n], sm.tags(0)[:n])
        cfg = bench.workload_config(m, None)
        assert "before eviction" in cfg["state"]
        assert "state" not in bench.workload_config(base, None)
    with pytest.raises(KeyError):
        W.get("no-such-workload")


def test_packed_step_round_trips_every_field_through_one_buffer():
    """The end-to-end leg moves a step's inputs with one copy of a packed
    buffer: every field survives the copy, starts on a 256-byte boundary, and
    the views are what the library calls receive."""
    from mixed_precision_paged_thinkv_b200.runner import PackedStep, StepInputs
    g = torch.Generator().manual_seed(3)
    B, H, d, Hq = 5, 2, 64, 8
    src = StepInputs(seqs=torch.arange(B, dtype=torch.int32),
                     pos=torch.randint(0, 1000, (B,), dtype=torch.int32, generator=g),
                     tags=torch.randint(0, 3, (B,), dtype=torch.uint8, generator=g),
                     k=torch.randn(B, H, d, generator=g).half(),
                     v=torch.randn(B, H, d, generator=g).half(),
                     budgets=torch.randint(1, 50, (B,), dtype=torch.int32, generator=g),
                     q=torch.randn(B, Hq, d, generator=g).half())
    host = PackedStep(src, "cpu").fill(src)
    dev = PackedStep(src, "cpu")
    dev.buf.copy_(host.buf)
    base = dev.buf.data_ptr()
    for f in StepInputs.FIELDS:
        a, b = getattr(src, f), getattr(dev.inputs, f)
        assert b.dtype == a.dtype and b.shape == a.shape and b.is_contiguous(), f
        assert torch.equal(a, b), f
        assert (b.data_ptr() - base) % PackedStep.ALIGN == 0, f
    assert host.nbytes() >= src.nbytes() and host.nbytes() % PackedStep.ALIGN == 0


def test_algorithmic_decode_bytes_counts_live_tokens_pages_and_rows():
    """Byte accounting on a hand-made state: sequence 0 has one 8-bit page with
    3 live slots and one 2-bit page with 16; sequence 1 has one 4-bit page with
    1 live slot.  d = 128, G = 64, 2 kv-heads, 4 q-heads, top-k on."""
    import numpy as np
    from mixed_precision_paged_thinkv_b200 import workloads as W
    w = W.scaled(W.WORKLOADS["tiny"], batch=2, num_q_heads=4, num_kv_heads=2, head_dim=128,
                 group_size=64, topk=32)
    def ent(page, cls, mask):
        return np.uint64(page | (cls << 32) | (mask << 48))
    table = np.zeros((2, 4), dtype=np.uint64)
    table[0, 0] = ent(7, 0, 0b111)
    table[0, 1] = ent(3, 2, 0xFFFF)
    table[1, 2] = ent(5, 1, 0b1000)
    live = np.zeros((2, 4), dtype=np.uint64)
    live[0, 0] = np.uint64(7 | (0 << 32) | (0 << 40))
    live[0, 1] = np.uint64(3 | (2 << 32) | (1 << 40))
    live[1, 0] = np.uint64(5 | (1 << 32) | (2 << 40))
    snap = {"num_live": np.array([2, 1], dtype=np.int32), "live_list": live, "table": table}
    total, by_class, pages = bench.algorithmic_decode_bytes(w, snap)
    assert by_class == [3, 1, 16] and pages == 3
    per = {8: 2 * 128 + 2 * 2 * 4, 4: 128 + 16, 2: 64 + 16}      # 272 / 144 / 80 B
    want = 2 * (3 * per[8] + 1 * per[4] + 16 * per[2])            # x kv-heads
    want += 3 * 16 + 2 * 8 + 2 * 2 * 4 * 128 * 2 + 2 * 4 * 4     # pages, seqs, Q+O, mass
    assert total == want


def test_compaction_bytes_counts_each_live_token_once_each_way():
    import bench
    from mixed_precision_paged_thinkv_b200 import workloads as W
    w = W.WORKLOADS["r1-llama-8b"]          # 8 kv-heads, d 128, G 64, bits 8/4/2
    # per (token, head): 272 / 144 / 80 bytes at 8 / 4 / 2 bits
    assert bench.compaction_bytes(w, [10, 0, 0]) == 2 * 10 * 8 * 272
    assert bench.compaction_bytes(w, [1, 2, 3]) == 2 * 8 * (272 + 2 * 144 + 3 * 80)

"""bench.py's host-side logic on the CPU: byte accounting, the traffic record, the max-over-ranks
timing across two gloo ranks, and the reference arm's JSON line."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import workloads as W


def test_step_bytes_counts_live_tokens_q_out_table_and_lengths():
    wl = W.custom(seed=1, num_seqs=3, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16, lens=[1, 16, 40])
    st = wl.steps[0]
    kv, alg = bench.step_bytes(wl, st)
    assert kv == (1 + 16 + 40) * 2 * 64 * 2 * 2
    assert alg == kv + 2 * 3 * 4 * 64 * 2 + 4 * (1 + 1 + 3) + 4 * 3


def test_job_rate_is_whole_job_over_slowest_rank():
    # 2 ranks x 1 GB per step x 10 steps in 20 ms (the slower rank) = 1000 GB/s
    assert bench.job_rate_gbs(10**9, 2, 10, 20.0) == pytest.approx(1000.0)


def test_traffic_record_requires_matching_kernel_sources(tmp_path, monkeypatch):
    val, note = bench.recorded_traffic("llama2_7b_decode")
    assert val is None or val > 0
    fake = tmp_path / "profiles"
    fake.mkdir()
    (tmp_path / "k.cuh").write_text("kernel v1")
    import hashlib
    rec = {"kernel_sources": ["k.cuh"], "kernel_sources_sha256": hashlib.sha256(b"kernel v1").hexdigest(),
           "workloads": {"w": {"kernel": "k", "dram_bytes_per_launch": 123, "how": "test"}}}
    (fake / "decode_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("w")[0] == 123
    assert bench.recorded_traffic("other")[0] is None
    (tmp_path / "k.cuh").write_text("kernel v2")
    assert bench.recorded_traffic("w") == (None, "kernel changed since the ncu capture")


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 5.0 - rank]  # rank 1 is slower on the first figure, faster on the second
        out[rank] = bench.max_over_ranks(local)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == [11.0, 5.0] and out[1] == [11.0, 5.0]


def test_reference_arm_prints_the_contract_line(capsys, monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "tiny_decode",
                                      "--steps", "2", "--warmup", "1"])
    assert bench.main() == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["value"] > 0 and line["higher_is_better"] is True and line["steps"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    """Under torchrun the reference arm runs on rank 0 alone; the other ranks exit 0 without work or output."""
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "tiny_decode", "--gpus", "2",
                                      "--steps", "2", "--warmup", "1"])
    assert bench.main() == 0
    assert capsys.readouterr().out.strip() == ""


def test_flush_rule_and_note():
    l2 = 126 * 10**6
    assert bench.flush_needed("auto", 67 * 10**6, l2)        # a shared-prefix step fits in L2: flush
    assert not bench.flush_needed("auto", 1_200 * 10**6, l2)  # the Llama-2 batch streams 10x the L2
    assert bench.flush_needed("on", 10**10, l2) and not bench.flush_needed("off", 1, l2)
    assert "flushed" in bench.l2_note(True, 10**6, l2, 512 * 2**20)
    assert "no flush" in bench.l2_note(False, 10**9, l2, 512 * 2**20)


def test_summary_of_per_iteration_times():
    s = bench.summarize_ms([0.010] * 8 + [0.020, 0.030])
    assert s["median_us"] == pytest.approx(10.0) and s["n"] == 10
    assert s["p10_us"] <= s["median_us"] <= s["p90_us"]
    assert s["mean_us"] == pytest.approx(13.0)


def test_shared_prefix_distinct_bytes_below_logical():
    wl = W.shared_prefix()
    st = wl.steps[1]
    kv, _ = bench.step_bytes(wl, st)
    uniq = W.unique_kv_bytes(st, wl.num_kv_heads, wl.head_dim, wl.block_size)
    assert uniq < kv / 3  # 8 tables name each prefix block


def test_cascade_traffic_record_has_its_own_sources(tmp_path, monkeypatch):
    import hashlib
    fake = tmp_path / "profiles"
    fake.mkdir()
    (tmp_path / "a.cuh").write_text("split kernel")
    (tmp_path / "c.cuh").write_text("cascade kernel v1")
    rec = {"kernel_sources": ["a.cuh"], "kernel_sources_sha256": hashlib.sha256(b"split kernel").hexdigest(),
           "workloads": {"w": {"kernel": "split", "dram_bytes_per_launch": 10, "how": "t"}},
           "cascade": {"kernel_sources": ["c.cuh"],
                       "kernel_sources_sha256": hashlib.sha256(b"cascade kernel v1").hexdigest(),
                       "workloads": {"w": {"kernel": "partial", "dram_bytes_per_launch": 20, "how": "t"}}}}
    (fake / "decode_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("w")[0] == 10
    assert bench.recorded_traffic("w", "cascade")[0] == 20
    (tmp_path / "c.cuh").write_text("cascade kernel v2")  # only the cascade record goes stale
    assert bench.recorded_traffic("w", "cascade") == (None, "kernel changed since the ncu capture")
    assert bench.recorded_traffic("w")[0] == 10
    assert bench.recorded_traffic("w", "missing")[0] is None


def test_committed_cascade_traffic_record_matches_the_sources():
    val, note = bench.recorded_traffic("shared_prefix_step", "cascade")
    assert val is not None, note
    wl = W.shared_prefix()
    uniq = W.unique_kv_bytes(wl.steps[0], wl.num_kv_heads, wl.head_dim, wl.block_size)
    assert uniq < val < 1.1 * uniq  # the shared tiles cross HBM once per group


def test_bench_decodes_through_the_cascade_only_when_groups_are_found():
    import paged_kv_cache_457_b200 as pa
    wl = W.shared_prefix()
    st = wl.steps[0]
    g = pa.find_prefix_groups(st.block_tables, st.context_lens, wl.block_size)
    assert g.num_groups == 8 and set(np.diff(g.offsets).tolist()) == {8} and set(g.prefix_blocks.tolist()) == {64}
    assert bench.cascade_wanted("auto", g.num_groups, 0)
    assert not bench.cascade_wanted("auto", g.num_groups, 256)  # a fixed partition is pa_decode's parameter
    assert not bench.cascade_wanted("off", g.num_groups, 0)
    tiny = W.tiny()
    g0 = pa.find_prefix_groups(tiny.steps[0].block_tables, tiny.steps[0].context_lens, tiny.block_size)
    assert g0.num_groups == 0 and not bench.cascade_wanted("auto", 0, 0)
    assert bench.cascade_wanted("on", 0, 0)

"""bench.py's multi-rank host logic on CPU: world-size-2 gloo ranks, each an
independent replica; the timed region is the max over ranks and the work
and units are summed (weak scaling, no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, world, rank)
        elapsed, units, work = bench.aggregate(10.0 + 5 * rank, 64.0, 1e9 * (rank + 1))
        bench.barrier()
        q.put((rank, elapsed, units, work))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, elapsed, units, work in got:
        assert elapsed == 15.0                 # max over ranks
        assert units == 128.0                  # sum over ranks
        assert work == 3e9


def test_single_process_aggregation_is_identity():
    import bench
    assert bench.aggregate(3.5, 7, 11) == (3.5, 7, 11)


def test_reference_arm_only_rank0_prints(capsys, monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.run_reference(type("A", (), {"workload": "tiny_decode_f32", "steps": 1, "warmup": 3,
                                       "ref_seqs": 1, "ref_items": 8})())
    assert capsys.readouterr().out == ""


def test_reference_arm_line_shape(capsys, monkeypatch):
    import json

    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    bench.run_reference(type("A", (), {"workload": "tiny_decode_f32", "steps": 2, "warmup": 3,
                                       "ref_seqs": 2, "ref_items": 8})())
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_reference_arm_cache_append_line(capsys, monkeypatch):
    """The cache-append workload's reference arm: the oracle's row copy of a full-cache
    scatter (here of a small decode batch standing in for the Llama-2-7B one)."""
    import json

    import numpy as np

    import bench
    from paged_kv_cache_380_b200 import workloads as W
    small = W.decode_case(name="small_c2", config_index=1, batch=3, num_q_heads=4, num_kv_heads=4, head_dim=128,
                          page_size=16, dtype="bf16", context_lens=np.array([17, 64, 300]))
    monkeypatch.setattr(W, "llama2_7b_mha_decode", lambda **kw: small)
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    bench.run_reference(type("A", (), {"workload": "kv_cache_write_full", "steps": 2, "warmup": 3,
                                       "ref_seqs": 1, "ref_items": 8})())
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["dtype"] == "u8" and line["config"]["workload"] == "kv_cache_write_full"
    assert line["cpu_baseline"]["kind"] == "oracle" and "381 rows" in line["cpu_baseline"]["sample"]


def test_cpu_baseline_reports_all_cores_and_one_thread():
    """cpu_baseline times the oracle twice: on all host threads and on one."""
    import numpy as np

    import bench
    import oracle
    from paged_kv_cache_380_b200 import workloads as W
    threads = oracle.max_threads()
    dec = W.tiny_decode_f32()
    step = type("S", (), {"case": dec, "kind": "decode", "int8": False, "has_new": False,
                          "decode_bytes": 1e6})()
    got = bench.cpu_baseline(step, budget_s=0.2)
    assert got["cores"] == threads and got["value"] > 0
    assert got["single_thread"]["cores"] == 1 and got["single_thread"]["value"] > 0
    assert oracle.max_threads() == threads                 # thread count restored
    pre = W.prefill_case(name="cpu_baseline_prefill", config_index=900, num_seqs=2, num_q_heads=4,
                         num_kv_heads=2, head_dim=128, page_size=16, dtype="bf16", shared_prefix=16,
                         chunk_lens=np.array([20, 9]), private_prefix=0)
    step = type("S", (), {"case": pre, "kind": "prefill", "work": 1e9})()
    got = bench.cpu_baseline(step, budget_s=0.2)
    assert got["unit"] == "TFLOP/s" and got["single_thread"]["cores"] == 1
    assert oracle.max_threads() == threads


def test_traffic_figures_belong_to_the_current_kernels():
    """Every DRAM-traffic figure bench.py can attach was captured on the kernel sources now in
    the tree (bench.py drops a figure whose source hash differs; this keeps none stale)."""
    import bench
    kind_of = {"llama2_7b_mha_decode": "decode", "llama2_70b_gqa_decode": "decode",
               "long_ctx_split_kv_int8": "decode", "chunked_prefill_shared_prefix": "prefill",
               "kv_cache_write_full": "scatter"}
    assert set(bench.TRAFFIC) == set(kind_of)
    for workload, tr in bench.TRAFFIC.items():
        assert tr["bytes"] > 0
        assert tr["kernel_sha"] == bench.kernel_sha(kind_of[workload]), workload

"""The multi-rank parts of bench.py on CPU: two gloo ranks, max-over-ranks
timing and whole-job aggregation (no GPU)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [3.0, 5.0][rank]  # the slower rank decides
        m = bench.reduce_max(ms, world, "cpu")
        bench.barrier(world)
        out[rank] = m
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == 5.0
    # each rank did its own 1e12-FLOP step; the job's rate uses the slowest rank
    assert bench.whole_job_tflops(1e12, world, 5.0) == pytest.approx(400.0)
    assert bench.whole_job_tflops(1e12, 1, 5.0) == pytest.approx(200.0)


def test_json_labels_follow_the_workload():
    from block_sparse_full_b200.inputs import WORKLOADS
    f32 = WORKLOADS["f32_T1024_d64"]
    assert f32.dtype == "f32"
    assert "planted" not in bench.data_description(f32)
    assert "/sqrt(d)" not in bench.data_description(f32)  # config 1 draws plain N(0,1)
    assert "hot key blocks" in bench.data_description(WORKLOADS["bf16_T8192_H16_hot"])
    assert "sink" in bench.data_description(WORKLOADS["bf16_T65536_H8_sink"])
    assert "planted" not in bench.data_description(WORKLOADS["bf16_B4_H32_T4096_train"])


def test_ncu_traffic_only_for_the_captured_workload_and_source(tmp_path, monkeypatch):
    import json
    table = {"k": {"sources": ["fwd_tc.cu"], "source_sha": bench.source_sha("fwd_tc.cu"),
                   "dram_bytes_per_launch": 123, "workload": "bf16_T8192_H16_hot (B1 H16 ...)"},
             "stale": {"sources": ["fwd_tc.cu"], "source_sha": "0" * 16,
                       "dram_bytes_per_launch": 456, "workload": "bf16_T8192_H16_hot"}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(table))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_sha", lambda *n: table["k"]["source_sha"])
    assert bench.ncu_traffic("k", "bf16_T8192_H16_hot") == 123
    assert bench.ncu_traffic("k", "bf16_T16384_H16_sweep") is None  # another workload
    assert bench.ncu_traffic("stale", "bf16_T8192_H16_hot") is None  # source changed since
    assert bench.ncu_traffic("missing", "bf16_T8192_H16_hot") is None


def test_both_arms_print_the_same_config_keys():
    from block_sparse_full_b200.inputs import WORKLOADS
    w = WORKLOADS["bf16_T8192_H16_hot"]
    ours = bench.workload_config(w, 2, "replicas x2")
    ref = bench.workload_config(w, 1, "oracle")
    assert set(ours) == set(ref)
    assert ours["workload"] == ref["workload"] == w.name
    assert ours["global_batch"] == 2 * w.B and ref["global_batch"] == w.B


def test_roofline_peak_follows_the_timed_region():
    # a short region runs at the clocks of the burst GEMM measurement, a long
    # one under the power cap like the sustained loop
    assert bench.roofline_peak(26.0, 1645.6, 1387.7)[0] == 1645.6
    assert "burst" in bench.roofline_peak(26.0, 1645.6, 1387.7)[1]
    assert bench.roofline_peak(2500.0, 1645.6, 1387.7)[0] == 1387.7


def test_gpus_flag_must_match_the_launch(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "2", "--impl", "reference"])

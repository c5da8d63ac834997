"""Host-side logic of the benchmark's multi-process launch (no GPU).

The path does not shard (replicas only): N ranks run independent replicas, the
job's time is the slowest rank's (max over ranks), and the reference arm runs
on rank 0 alone. These run as world-size-2 gloo processes on the CPU."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=2)
    try:
        v = bench.max_over_ranks(1.5 + rank, 2, "cpu")
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
        f.write(repr(v))


def test_max_over_ranks_gloo(tmp_path):
    mp.spawn(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=2, join=True)
    got = [float(open(tmp_path / f"r{r}.txt").read()) for r in range(2)]
    assert got == [2.5, 2.5]


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25


def _run_reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "tiny-ffn", "--gpus", str(world), "--steps", "1",
                           "--warmup", "1", "--cpu-seconds", "0.5"],
                          env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_rank0_prints_one_line():
    r = _run_reference(0, 2)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is False
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_reference(1, 2)
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_launches_per_call_counts_kernels_per_pass():
    # per pass: Stage 1 and one Stage-2 kernel (CUDA cores) or two (tensor-core
    # union engine: automatic for 8-token passes, and for 4-token passes when
    # d_model >= 8192, whose passes hold at most 4 tokens)
    sys.path.insert(0, ROOT)
    import argparse

    import bench

    def n(engine, d, batch):
        return bench.launches_per_call(argparse.Namespace(engine=engine), d, batch)

    assert n("auto", 4096, 1) == 2 and n("auto", 4096, 2) == 2 and n("auto", 4096, 4) == 2
    assert n("auto", 4096, 8) == 3 and n("auto", 4096, 5) == 3      # one pass of 8 slots
    assert n("simt", 4096, 8) == 2 and n("tc", 4096, 4) == 3 and n("tc", 4096, 2) == 2
    assert n("auto", 8192, 4) == 3 and n("auto", 8192, 16) == 4 * 3  # passes of 4
    assert n("simt", 8192, 16) == 4 * 2


def test_stage2_traffic_scaled_to_the_mean_token():
    # the committed Stage-2 summary holds one token's traffic and algorithmic
    # bytes; the bench reports it scaled to the mean token's bytes, and only
    # for the workload and batch the capture covers
    sys.path.insert(0, ROOT)
    import bench
    fields = bench.summary_fields(os.path.join(ROOT, "profiles", "k_stage2_qwen3-8b-ffn_b1.md"))
    traffic = float(fields["dram bytes per launch (read + write)"])
    captured = float(fields["algorithmic bytes of the captured launch"].split()[0])
    got = bench.traffic_from_summary(fields, 90537600.0)
    assert got is not None and abs(got - traffic * 90537600.0 / captured) < 1.0
    assert bench.traffic_from_summary({}, 1.0) is None
    assert bench.stage2_traffic("qwen3-8b-ffn", 8, 1.0) is None
    assert bench.stage2_traffic("large-ffn", 1, 1.0) is None


def test_stamp_phases_add_up_to_the_call():
    # two adjacent calls' stamps (ns): stage1 + stage2 is the call, and each
    # sub-phase is the difference of its slots
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    NONE = -1
    a = np.zeros(16, dtype=np.int64)
    b = np.zeros(16, dtype=np.int64)
    base = 10_000_000
    a[[0, 1, 2, 3, 4, 5, 6]] = base + np.array([0, 1000, 1200, 2000, 6000, 6500, 7500])
    a[[8, 9, 10, 11, 12, 13, 14, 15]] = base + np.array([500, 8000, 8100, 8900, 9500, 9800,
                                                         24000, 25000])
    b[[0, 1]] = base + np.array([24500, 26000])
    b[8] = b[9] = b[12] = NONE
    st = np.stack([a, b])
    ph = bench.stamp_phases(st, [0, 1], {0: 0, 1: 1})
    assert ph["pairs"] == 1
    assert abs(ph["stage1"] - 7.0) < 1e-9 and abs(ph["stage2"] - 18.0) < 1e-9
    assert abs(ph["call"] - (ph["stage1"] + ph["stage2"])) < 1e-9
    assert abs(ph["s1_prologue"] - 1.0) < 1e-9 and abs(ph["s1_stream"] - 4.0) < 1e-9
    assert abs(ph["s1_exit_to_s2_go"] - 0.5) < 1e-9
    assert abs(ph["s2_list"] - 0.9) < 1e-9 and abs(ph["s2_first_data"] - 0.9) < 1e-9
    assert abs(ph["s2_stream_window"] - 14.5) < 1e-9 and abs(ph["s2_tail"] - 1.0) < 1e-9
    assert abs(ph["s2_exit_to_next_s1_go"] - 1.0) < 1e-9
    # a call whose Stage 2 left no stamps (slots still at their reset values) is skipped
    st2 = st.copy()
    st2[0, 9] = NONE
    assert bench.stamp_phases(st2, [0, 1], {0: 0, 1: 1})["pairs"] == 0

"""Host-side logic of bench.py on the CPU: algorithmic bytes and FLOPs of each
workload against hand-derived values, L2 rotation sizing, and the
multi-process (torch.distributed, gloo, world size 2) reduction of elapsed time
and token counts that a multi-GPU run uses.  The path shards as independent
data-parallel replicas, so there is no data-path collective to test, only the
timing / throughput aggregation."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from gather_matmul_b200 import workloads as W


def test_algorithmic_bytes_decode_q_proj_by_hand():
    p = W.config(2)[0]                       # T=256 all active, U=32 slots, D=D_out=4096, r=16
    by = bench.algorithmic_bytes(p)
    Ta, U, D, r, T = 256, 32, 4096, 16, 256
    assert bench.active_stats(p) == (Ta, U)
    assert by["shrink"] == Ta * D * 2 + U * r * D * 2 + 4 * T + 4 * T * r
    assert by["expand"] == 4 * T + 4 * Ta * r + U * D * r * 2 + 2 * Ta * D * 2
    assert by["group"] == 8 * T
    assert bench.algorithmic_flops(p) == 2 * Ta * r * D * 2


def test_algorithmic_bytes_segments_and_slices():
    ss, sa = np.array([0, 100, 100, 260, 300]), np.array([2, 0, -1, 1])
    p = W.make_problem("s", W.BF16, T=300, D=512, r=32, S=3, d_out=[256, 128], seed=1,
                       segments=(ss, sa))
    Ta, U = bench.active_stats(p)
    assert (Ta, U) == (100 + 40, 2)            # the empty segment and the -1 segment drop out
    by = bench.algorithmic_bytes(p)
    assert by["group"] == 0
    assert by["expand"] == 4 * 300 + sum(4 * Ta * 32 + U * o * 32 * 2 + 2 * Ta * o * 2
                                         for o in (256, 128))


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5])
def test_workload_bytes_are_positive_and_consistent(n):
    for p in W.config(n):
        by = bench.algorithmic_bytes(p)
        assert by["step"] == by["shrink"] + by["expand"] + by["group"] > 0
        assert bench.call_bytes(p, "fused") == by["shrink"] + by["expand"]


def test_kernel_names_follow_the_dispatch_rules():
    # decode q_proj: T = 256 < 16 * 32 -> CUDA-core item kernels when not fused
    p2 = W.config(2)[0]
    assert bench.kernels_of(p2, "shrink", False) == ["shrink_items_kernel"]
    assert bench.kernel_calls(p2, True) == ["fused"]
    assert bench.kernels_of(p2, "fused", True) == ["bgmv_fused_kernel"]
    # large mixed: r = 32, T = 4096 >= 16 * 128 -> grouped tensor-core kernels
    p5 = W.config(5)[0]
    assert bench.grouped_tc(p5)
    assert bench.kernel_calls(p5, False) == ["group", "shrink", "expand"]
    assert bench.kernels_of(p5, "expand", False) == ["sgmv_expand_tc_kernel"]
    # prefill segments on tensor cores; rank 8 segments on the item kernels
    p4 = W.config(4)[0]
    assert bench.kernels_of(p4, "shrink", False) == ["sgmv_shrink_tc_kernel"]
    q = W.make_problem("s", W.F16, T=64, D=64, r=8, S=2, d_out=[64], seed=1,
                       segments=(np.array([0, 30, 64]), np.array([0, 1])))
    assert bench.kernels_of(q, "expand", False) == ["segment_items_kernel", "expand_items_kernel"]


def test_call_flops_and_e2e_window():
    p = W.config(2)[0]
    assert bench.call_flops(p, "fused") == bench.algorithmic_flops(p)
    assert bench.call_flops(p, "shrink") + bench.call_flops(p, "expand") == \
        bench.algorithmic_flops(p)
    # at least K steps, and at least 100 ms at the estimated step time
    assert bench.e2e_steps_for(1e-3, 20) == 100
    assert bench.e2e_steps_for(1e-1, 20) == 20
    assert bench.e2e_steps_for(1e-9, 20) == 20000      # capped


def test_rotation_sets_cover_three_l2():
    assert bench.rotation_sets(15e6) * 15e6 >= 3 * bench.L2_BYTES
    assert bench.rotation_sets(1e12) == 2          # never fewer than two sets
    assert bench.rotation_sets(1) == 64            # capped


def test_profile_traffic_requires_matching_sources(tmp_path, monkeypatch):
    import json
    f = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(f))
    k = "bgmv_fused_kernel"
    assert bench.profile_traffic(k) is None
    f.write_text(json.dumps({"kernels": {k: {"source_hash": "stale", "dram_bytes_per_launch": 5}}}))
    assert bench.profile_traffic(k) is None
    f.write_text(json.dumps({"kernels": {k: {"source_hash": bench.kernel_source_hash(k),
                                             "dram_bytes_per_launch": 5}}}))
    assert bench.profile_traffic(k) == 5
    assert bench.profile_traffic("not_a_kernel") is None
    # each kernel's figure follows its own sources only
    assert bench.kernel_source_hash(k) != bench.kernel_source_hash("sgmv_expand_tc_kernel")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        assert (ws, r, local) == (world, rank, rank)
        cpu = torch.device("cpu")
        # every rank serves its own batch; the job is timed by the slowest rank
        elapsed = [0.5, 0.8][rank]
        tokens = [1000, 1000][rank]
        el_max = bench.max_over_ranks(elapsed, ws, cpu)
        tok = bench.sum_over_ranks(tokens, ws, cpu)
        bench.barrier(ws)
        q.put((rank, el_max, tok, tok / el_max))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for _, el, tok, val in res:
        assert el == 0.8 and tok == 2000 and val == pytest.approx(2500.0)


def test_single_rank_helpers_are_identity():
    cpu = torch.device("cpu")
    assert bench.max_over_ranks(1.25, 1, cpu) == 1.25
    assert bench.sum_over_ranks(7, 1, cpu) == 7
    assert bench.aggregate([100, 300], 2.0) == 200.0


def _run_bench(args, env_extra=None):
    import json
    import subprocess
    import sys
    env = dict(os.environ)
    env.update(env_extra or {})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    return [json.loads(l) for l in lines]


def test_reference_arm_line():
    (line,) = _run_bench(["--impl", "reference", "--steps", "3", "--warmup", "3",
                          "--reference-seconds", "2"], {"WORLD_SIZE": "1", "RANK": "0"})
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["steps"] == 3
    assert line["higher_is_better"] is True and line["vs_baseline"] is None


def test_reference_arm_other_ranks_print_nothing():
    assert _run_bench(["--impl", "reference", "--steps", "3", "--warmup", "3"],
                      {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"}) == []

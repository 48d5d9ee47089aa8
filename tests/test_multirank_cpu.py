"""The N > 1 host path of bench.py (independent replicas, one per GPU) on CPU
ranks over gloo: the barrier, the max over ranks that times the job, the
whole-job throughput, per-rank inputs, and the reference arm under the
launcher (rank 0 alone runs and prints)."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from convolved_logit_attention_b200.workloads import WORKLOADS, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        # each rank reports its own (rank-dependent) time; all must see the max
        m = bench.dist_max(1.5 + rank, world, torch.device("cpu"))
        with open(os.path.join(out_dir, "rank%d.txt" % rank), "w") as f:
            f.write(repr(m))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_barrier_and_max_over_ranks_gloo(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        assert float((tmp_path / ("rank%d.txt" % r)).read_text()) == 2.5


def test_replica_throughput_counts_every_rank_and_the_slowest_time():
    one = bench.replica_tflops(1, 1.74e11, 10, 5.0)
    assert abs(one - 1.74e11 * 10 / 5e-3 / 1e12) < 1e-9
    assert bench.replica_tflops(4, 1.74e11, 10, 5.0) == 4 * one
    assert bench.replica_tflops(2, 1.74e11, 10, 10.0) == one     # slowest rank halves it


def test_each_replica_draws_its_own_inputs():
    w = WORKLOADS["tiny_f32"]
    a, b = make_inputs(w, seed=w.seed + 0), make_inputs(w, seed=w.seed + 1)
    assert a["q"].shape == b["q"].shape and not np.array_equal(a["q"], b["q"])


def test_reference_arm_under_the_launcher_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node",
           "2", "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--workload", "tiny_f32", "--steps", "1",
           "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1                      # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 2


def test_reference_arm_times_a_composition():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_f32",
           "--compose", "repeat", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][0])
    assert d["config"]["composition"] == "repeat" and d["value"] > 0


@pytest.mark.parametrize("name", ["repeat", "exact_both_pre", "conv3d_exact_mix"])
def test_oracle_units_are_slices_of_the_composed_forward(name):
    # The CPU-baseline sample cuts (batch, head-group) units out of the
    # workload, post-softmax weights included; each unit's oracle output
    # is the matching slice of the whole problem's.
    import oracle
    from convolved_logit_attention_b200.workloads import COMPOSITIONS, composed_inputs
    w = WORKLOADS["tiny_f32"]
    x = composed_inputs(w, name)
    flops = w.composition_flops(COMPOSITIONS[name])
    units, f = bench.oracle_sample(w, x, 2, flops)
    assert f == 2 * flops // (w.B * w.G)
    full = oracle.forward_composed(x["q"], x["k"], x["v"], x["w_kq"], x["w_head"], x["w_kq_post"],
                                   x["w_head_post"], x["gn_weight"], x["gn_bias"], w.depth_scale,
                                   w_head_pre=x["w_head_pre"], exact_mask=x["exact_mask"],
                                   w_kq_3d=x["w_kq_3d"])
    for g, u in enumerate(units):
        part = bench.run_oracle_unit(u, w)
        cs = slice(g * w.c_h * w.d, (g + 1) * w.c_h * w.d)
        np.testing.assert_array_equal(part[0], full[0, :, cs])

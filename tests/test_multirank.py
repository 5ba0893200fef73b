"""The multi-GPU path of bench.py (independent replicas, weak scaling; or one job
sharded into contiguous (b, kv-head) slices, strong scaling) on CPU ranks.

Two gloo ranks on 127.0.0.1 run bench.py's per-rank pieces: each rank seeds its own
replica, the timings are reduced to the max over ranks (the slowest rank sets the
job's time), the whole-job throughput counts every rank's work, and the reference
arm runs on rank 0 only.  No GPU and no collective on the data path are involved.
"""
import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    import bench
    from attn_inputs import WORKLOADS, make_inputs
    w = WORKLOADS["single_head_n256_d64"]
    seed = bench.rank_seed(w, rank)
    x = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=seed, device="cpu", with_grad=False)
    # rank r "measured" (10 + r) ms total and (3 - r) ms forward
    total, fwd = bench.max_over_ranks([10.0 + rank, 3.0 - rank], dist, "cpu")
    res = {"rank": rank, "seed": seed, "total": total, "fwd": fwd, "q0": float(x["q"].float()[0, 0, 0, 0])}
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest_and_seed_their_own_replicas(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["total"] == 11.0 and r["fwd"] == 3.0
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["q0"] != res[1]["q0"]


def test_weak_scaling_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.weak_scaling_tflops(1e12, 1, 10.0)
    assert one == pytest.approx(100.0)
    assert bench.weak_scaling_tflops(1e12, 8, 10.0) == pytest.approx(8 * one)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload = "single_head_n256_d64"
        steps = 1
        warmup = 0
        gpus = 2

    bench.run_reference(Args, rank=1, world=2)
    assert capsys.readouterr().out == ""
    bench.run_reference(Args, rank=0, world=2)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    # the same keys as the main arm's line, plus the baseline description
    for key in ("metric", "unit", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    # ms_per_step is one whole step of the workload at the measured rate
    f, fb = bench.step_flops(bench.WORKLOADS[Args.workload])
    assert abs(line["ms_per_step"] - (f + fb) / (line["value"] * 1e12) * 1e3) <= 1e-9 * line["ms_per_step"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_shard_units_partition_the_job_contiguously():
    sys.path.insert(0, ROOT)
    import bench
    for total in (1, 7, 32, 128, 1000):
        for world in (1, 2, 3, 4, 8):
            spans = [bench.shard_units(total, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def _shard_rank(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    import numpy as np
    import torch.distributed as dist
    from attn_inputs import Workload, make_inputs, to_f64
    from oracle import reference as ref
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = Workload("tiny", 3, 4, 2, 9, 4, True, "fwd", seed=77)
        full = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=w.seed, with_grad=False)
        views, units = bench.shard_views(full, w, rank, world)
        o, lse = ref.ref_fwd(*(to_f64(views[n]) for n in ("q", "k", "v")), 0.5, w.causal)
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_shard_views_map_each_rank_to_its_heads(tmp_path, world):
    """Each rank's contiguous slice of the (b, kv-head) units, attended on its own, gives
    exactly its heads' rows of the whole job (GQA groups stay together)."""
    import numpy as np
    import torch.multiprocessing as mp
    from attn_inputs import make_inputs, to_f64
    from oracle import reference as ref
    mp.start_processes(_shard_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    full = make_inputs(3, 4, 2, 9, 4, seed=77, with_grad=False)
    o_ref, _ = ref.ref_fwd(*(to_f64(full[n]) for n in ("q", "k", "v")), 0.5, True)
    flat = o_ref.reshape(1, 12, 9, 4)
    got = np.concatenate([np.load(tmp_path / f"o{r}.npy") for r in range(world)], axis=1)
    np.testing.assert_array_equal(got, flat)

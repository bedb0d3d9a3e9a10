"""Multi-rank host logic of the benchmark on CPU, world size 2 over gloo.

On GPUs every rank runs its own batch (weak scaling) and the only cross-rank
operations are a barrier and the max-reduction of the timed interval, plus,
when asked for, the data-parallel exchange of dW and dE (all-reduce or
reduce-scatter); these tests run exactly those pieces with the gloo backend
on 127.0.0.1.
"""
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

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from lm_head_loss_junction_b200 import workloads as wl
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench._dist_env()
        assert (ws, r, local) == (world, rank, rank)
        # every rank reports the max of the ranks' intervals
        mx = bench._max_over_ranks(10.0 + 5.0 * rank, ws, torch.device("cpu"))
        # each rank draws its own batch (seed offset by rank)
        import dataclasses
        cfg = dataclasses.replace(wl.small_variant(wl.CONFIGS["main3"], batch=1, seq=64, V=256),
                                  seed=wl.CONFIGS["main3"].seed + rank)
        d = wl.make_inputs(cfg, with_heads=False, with_tables=False)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": mx, "x": d.x.tolist()}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_reduce_and_distinct_batches(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    assert r0["max"] == r1["max"] == 15.0
    assert not np.array_equal(r0["x"], r1["x"]), "ranks must draw different batches"


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, WORLD_SIZE="2", MASTER_ADDR="127.0.0.1")
    args = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny3",
            "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-tokens", "16"]
    outs = []
    for rank in (0, 1):
        p = subprocess.run(args, env=dict(env, RANK=str(rank), LOCAL_RANK=str(rank)), capture_output=True,
                           text=True, timeout=300)
        assert p.returncode == 0, p.stderr[-2000:]
        outs.append([ln for ln in p.stdout.splitlines() if ln.strip()])
    assert len(outs[0]) == 1 and outs[1] == []
    line = json.loads(outs[0][0])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def _sync_main(rank, world, port, out_dir, mode):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(100 + rank)
        grads = [torch.randn(6, 4, generator=g), torch.randn(10, 2, generator=g)]   # a dW and a dE
        shards = bench.grad_shards(grads, world) if mode == "reduce_scatter" else None
        before = [t.clone() for t in grads]
        bench.grad_sync(grads, mode, world, shards)
        res = {"before": [t.tolist() for t in before]}
        res["after"] = [t.tolist() for t in grads] if mode == "allreduce" else [t.tolist() for t in shards]
        with open(os.path.join(out_dir, f"{mode}{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", ["allreduce", "reduce_scatter"])
def test_two_gloo_ranks_gradient_exchange(tmp_path, mode):
    port = _free_port()
    mp.start_processes(_sync_main, args=(2, port, str(tmp_path), mode), nprocs=2, join=True, start_method="spawn")
    r = [json.load(open(tmp_path / f"{mode}{k}.json")) for k in (0, 1)]
    for i in range(2):
        total = np.array(r[0]["before"][i]) + np.array(r[1]["before"][i])
        if mode == "allreduce":
            for k in (0, 1):
                np.testing.assert_allclose(r[k]["after"][i], total, rtol=1e-6)
        else:
            flat = total.reshape(-1)
            half = flat.size // 2
            np.testing.assert_allclose(r[0]["after"][i], flat[:half], rtol=1e-6)
            np.testing.assert_allclose(r[1]["after"][i], flat[half:], rtol=1e-6)


def test_gradient_exchange_is_a_no_op_on_one_rank():
    sys.path.insert(0, ROOT)
    import bench
    t = [torch.ones(3)]
    bench.grad_sync(t, "allreduce", 1)
    assert torch.equal(t[0], torch.ones(3))
    with pytest.raises(ValueError):
        bench.grad_shards([torch.ones(5)], 2)

"""Multi-rank path on the CPU (gloo, world size 2): the row shards cover the batch
exactly once, a rank's shard of the synthetic input equals the same rows drawn in one
process, sharded results gathered back equal the unsharded result, the timing
reduction takes the maximum over ranks, and the bench's reference arm under torchrun
prints one line from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

from structured_rotations_b200.shard import max_over_ranks, strong_shard, weak_shard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("total,world", [(0, 3), (1, 2), (7, 2), (65536, 8), (1000, 7), (5, 8)])
def test_strong_shards_cover_every_row_once(total, world):
    seen = np.zeros(total, dtype=int)
    sizes = []
    nxt = 0
    for r in range(world):
        start, count = strong_shard(total, world, r)
        assert start == nxt                      # contiguous, in rank order
        seen[start:start + count] += 1
        sizes.append(count)
        nxt = start + count
    assert nxt == total and np.all(seen == 1)
    assert max(sizes) - min(sizes) <= 1


def test_weak_shards_are_disjoint_blocks():
    blocks = [weak_shard(300, r) for r in range(4)]
    assert blocks == [(0, 300), (300, 300), (600, 300), (900, 300)]
    with pytest.raises(ValueError):
        strong_shard(10, 0, 0)
    with pytest.raises(ValueError):
        strong_shard(10, 2, 2)


def test_max_over_ranks_without_a_group_is_the_identity():
    assert max_over_ranks(3.25) == 3.25


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist
    import datetime
    sys.path.insert(0, ROOT)
    import workloads as W
    from oracle import harp_oracle as O
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        res = {"max": max_over_ranks(10.0 + rank, dist), "max_neg": max_over_ranks(-1.0 - rank, dist)}
        w = W.get("d5120")
        row0, rows = weak_shard(40, rank)
        enc = W.draw_encoded(w, row0, rows)
        theta = W.draw_theta(O.theta_count(w.schedule), w.theta_sigma, w.theta_seed)
        tr = O.Transform(O.make_plan(w.d, w.schedule, theta, sign_seed=w.sign_seed))
        y = tr.forward(W.decode_bf16(enc))
        gathered = [None] * world
        dist.all_gather_object(gathered, (row0, rows, y))
        if rank == 0:
            whole = np.concatenate([g[2] for g in sorted(gathered, key=lambda g: g[0])])
            enc_all = W.draw_encoded(w, 0, 40 * world)
            res["same_input"] = bool(np.array_equal(np.concatenate(
                [W.draw_encoded(w, g[0], g[1]) for g in gathered]), enc_all))
            res["same_output"] = bool(np.array_equal(whole, tr.forward(W.decode_bf16(enc_all))))
            res["rows"] = int(whole.shape[0])
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    assert r0["max"] == r1["max"] == 11.0
    assert r0["max_neg"] == r1["max_neg"] == -1.0
    assert r0["same_input"] and r0["same_output"] and r0["rows"] == 80


def test_bench_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["value"] > 0 and out["n_gpus"] == 2
    assert out["e2e"]["h2d_bytes_per_step"] == 0


def _two_sided_worker(rank, world, port, out_dir):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import workloads as W
    from oracle import harp_oracle as O
    from structured_rotations_b200.shard import two_sided_row_sharded
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        u_s, v_s = (8, 2, 4), (4, 2, 2)                       # n_out 64, n_in 16
        tu = O.Transform(O.make_plan(64, u_s, W.draw_theta(O.theta_count(u_s), 0.3, 5), sign_seed=6))
        tv = O.Transform(O.make_plan(16, v_s, W.draw_theta(O.theta_count(v_s), 0.3, 7), sign_seed=8))
        w = np.random.default_rng(11).standard_normal((64, 16))
        n = 64 // world
        w_local = torch.from_numpy(w[rank * n:(rank + 1) * n].copy())

        def row_fn(src, dst):
            dst.copy_(torch.from_numpy(tv.inverse(src.numpy())))

        def col_fn(src, dst):
            dst.copy_(torch.from_numpy(tu.inverse(src.numpy().T).T))

        out = two_sided_row_sharded(None, None, w_local, work_dtype=torch.float64, row_fn=row_fn, col_fn=col_fn)
        parts = [None] * world
        dist.all_gather_object(parts, out.numpy())
        if rank == 0:
            got = np.concatenate(parts)
            want = tu.inverse(tv.inverse(w).T).T                 # T_U^T W T_V
            with open(os.path.join(out_dir, "two_sided.json"), "w") as f:
                json.dump({"max_err": float(np.abs(got - want).max()), "shape": list(got.shape)}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_two_sided_row_sharded_exchange(tmp_path, world):
    """The row-sharded two-sided rotation (rows local, all-to-all, columns local,
    all-to-all back) on gloo ranks, with a float64 reference as each rank's compute,
    equals the single-process T_U^T W T_V."""
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_two_sided_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    r = json.load(open(tmp_path / "two_sided.json"))
    assert r["shape"] == [64, 16]
    assert r["max_err"] < 1e-12


def _grad_worker(rank, world, port, out_dir):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import workloads as W
    from oracle import harp_oracle as O
    from structured_rotations_b200.shard import grad_theta_sharded, strong_shard
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        sched = (8, 2, 4)
        plan = O.make_plan(64, sched, W.draw_theta(O.theta_count(sched), 0.3, 3), sign_seed=4)
        rng = np.random.default_rng(21)
        x, g = rng.standard_normal((37, 64)), rng.standard_normal((37, 64))
        r0, n = strong_shard(37, world, rank)

        def grad_fn(xl, gl):
            return torch.from_numpy(O.theta_grad(plan, xl.numpy(), gl.numpy()))

        got = grad_theta_sharded(None, torch.from_numpy(x[r0:r0 + n].copy()), torch.from_numpy(g[r0:r0 + n].copy()),
                                 grad_fn=grad_fn)
        parts = [None] * world
        dist.all_gather_object(parts, got.numpy())
        if rank == 0:
            want = O.theta_grad(plan, x, g)
            with open(os.path.join(out_dir, "grad.json"), "w") as f:
                json.dump({"max_err": float(max(np.abs(p_ - want).max() for p_ in parts)),
                           "scale": float(np.abs(want).max())}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_grad_theta_sharded_sums_over_ranks(tmp_path, world):
    """The calibration backward over row shards (each rank its rows' gradient, one
    all-reduce) gives every rank the gradient of all rows, on gloo ranks with a float64
    reference as each rank's compute."""
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_grad_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    r = json.load(open(tmp_path / "grad.json"))
    assert r["max_err"] <= 1e-12 * max(1.0, r["scale"])


def test_grad_theta_sharded_without_a_process_group_is_the_local_gradient():
    import torch
    from structured_rotations_b200.shard import grad_theta_sharded

    class FakePlan:
        def grad_theta(self, x, g):
            return (x * g).sum(dim=0)

    x, g = torch.arange(12.0).reshape(3, 4), torch.ones(3, 4)
    assert torch.equal(grad_theta_sharded(FakePlan(), x, g), (x * g).sum(dim=0))

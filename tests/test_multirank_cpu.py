"""Multi-rank host logic on CPU (gloo, world size 2).

The quantization path shards by rows with no data exchange (rows are
independent; the MoE group index is rebased per shard), and so does the W8A8
product that consumes the codes (weights replicated). These tests run two
gloo ranks that each quantize their shard with the CPU oracle, multiply it by
the weights and gather the results, and check the concatenations against one
unsharded run; and they run the benchmark's reference arm under torchrun with
two ranks.
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


def _worker(rank, world, port, out_path):
    sys.path.insert(0, ROOT)
    import oracle
    from token_dynamic_quantization_b200 import sharding, workloads

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rows, cols, experts = 203, 96, 6
        x = workloads.normal((rows, cols), torch.bfloat16, 0)
        smooth = workloads.uniform((experts, cols), torch.float32, 2, 0.5, 2.0)
        gi = workloads.moe_group_index(rows, experts, 3).numpy()
        start, end = sharding.row_range(rows, world, rank)
        local_gi = sharding.rebase_group_index(gi, start, end)
        y, s, _ = oracle.dynamic_quant(x[start:end], smooth=smooth, group_index=local_gi)
        # gather the shards (variable sizes: pad to the largest)
        n = torch.tensor([end - start])
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, n)
        cap = int(max(t.item() for t in sizes))
        yp = torch.zeros(cap, cols, dtype=torch.int8)
        sp = torch.zeros(cap, dtype=torch.float32)
        yp[: end - start] = torch.from_numpy(y)
        sp[: end - start] = torch.from_numpy(s)
        ys = [torch.zeros_like(yp) for _ in range(world)]
        ss = [torch.zeros_like(sp) for _ in range(world)]
        dist.all_gather(ys, yp)
        dist.all_gather(ss, sp)
        # the consumer shards the same way: each rank multiplies its own codes
        # (per-token scales) by the replicated int8 weights
        w = workloads.uniform((40, cols), torch.float32, 8, -127.0, 127.0).round().to(torch.int8).numpy()
        ws = workloads.uniform((40,), torch.float32, 9, 0.001, 0.02).numpy()
        pp = torch.zeros(cap, 40, dtype=torch.float32)
        pp[: end - start] = torch.from_numpy(oracle.w8a8_gemm(y, w, s, ws, out_dtype="f32"))
        ps = [torch.zeros_like(pp) for _ in range(world)]
        dist.all_gather(ps, pp)
        if rank == 0:
            y_all = torch.cat([ys[i][: sizes[i].item()] for i in range(world)]).numpy()
            s_all = torch.cat([ss[i][: sizes[i].item()] for i in range(world)]).numpy()
            p_all = torch.cat([ps[i][: sizes[i].item()] for i in range(world)]).numpy()
            y_ref, s_ref, _ = oracle.dynamic_quant(x, smooth=smooth, group_index=gi)
            p_ref = oracle.w8a8_gemm(y_ref, w, s_ref, ws, out_dtype="f32")
            ok = bool(np.array_equal(y_all, y_ref) and np.array_equal(s_all.view(np.uint32), s_ref.view(np.uint32))
                      and np.array_equal(p_all.view(np.uint32), p_ref.view(np.uint32)))
            with open(out_path, "w") as f:
                f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def test_row_range_covers_rows():
    from token_dynamic_quantization_b200 import sharding

    for rows in (0, 1, 7, 8192):
        for world in (1, 2, 3, 8):
            ranges = [sharding.row_range(rows, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == rows
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            assert max(e - s for s, e in ranges) - min(e - s for s, e in ranges) <= 1


def test_rebase_group_index():
    from token_dynamic_quantization_b200 import sharding

    gi = np.array([0, 40, 40, 100, 180, 300])
    assert list(sharding.rebase_group_index(gi, 100, 200)) == [0, 0, 0, 0, 80, 100]
    assert list(sharding.rebase_group_index(gi, 0, 50)) == [0, 40, 40, 50, 50, 50]


def test_two_gloo_ranks_match_unsharded(tmp_path):
    out = str(tmp_path / "result.txt")
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
    assert open(out).read() == "ok"


def test_bench_reference_arm_under_torchrun():
    """--impl reference under two ranks: rank 0 prints one JSON line, rank 1 exits 0."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3",
           "--cpu-seconds", "0.3", "--workload", "sym_int8_f16_64x1024"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def test_bench_gpus_n_starts_its_own_ranks():
    """`bench.py --gpus 2` started as one plain process re-runs itself under
    torch.distributed.run with two ranks: the line reports n_gpus 2."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "3",
           "--warmup", "3", "--cpu-seconds", "0.3", "--workload", "sym_int8_f16_64x1024"]
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    env["OMP_NUM_THREADS"] = "1"
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2


def test_bench_refuses_a_world_size_that_differs_from_gpus():
    """Under a launcher whose WORLD_SIZE is not --gpus, bench.py exits non-zero
    instead of timing the wrong number of ranks."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "3",
           "--warmup", "3", "--cpu-seconds", "0.3", "--workload", "sym_int8_f16_64x1024"]
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0", OMP_NUM_THREADS="1")
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert res.returncode != 0
    assert "WORLD_SIZE" in res.stderr

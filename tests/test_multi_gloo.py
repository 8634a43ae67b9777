"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): replicas need no data-path
collective; only rank 0 prints; timings are reduced with a max over ranks."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
        bench.barrier(world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29511
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 11.0, 1: 11.0}


def test_reference_arm_prints_once_under_torchrun():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", "29512", "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny",
           "--ref-rows", "4"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "ms/layer"
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_head_shard_partitions_every_head_once():
    import block_sparse_long_qk_b200 as fp
    for Hq, Hkv in ((32, 8), (28, 4), (8, 8), (6, 3)):
        for world in range(1, Hkv + 1):
            qh, kh = [], []
            for r in range(world):
                qs, ks = fp.head_shard(Hq, Hkv, r, world)
                qh += list(range(qs.start, qs.stop))
                kh += list(range(ks.start, ks.stop))
                G = Hq // Hkv
                assert qs.start == ks.start * G and qs.stop == ks.stop * G   # whole groups
            assert qh == list(range(Hq)) and kh == list(range(Hkv))
            sizes = [fp.head_shard(Hq, Hkv, r, world)[1].stop - fp.head_shard(Hq, Hkv, r, world)[1].start
                     for r in range(world)]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        fp.head_shard(32, 8, 0, 9)
    with pytest.raises(ValueError):
        fp.head_shard(30, 8, 0, 2)


def _split_worker(rank, world, port, q):
    """Rank r runs the oracle's whole path (pool, scores, keep sets, attention) on its head
    slice of one small layer; the slices are gathered over gloo."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import dataclasses
    import bench
    from block_sparse_long_qk_b200 import synthetic as S
    from _parity import OracleRun
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = dataclasses.replace(S.WORKLOADS["llama128k"], Hq=8, Hkv=4)
        inp = S.make_inputs(w, seed=5, seqlens=(700, 300))
        part = bench.shard_inputs(inp, rank, world)
        run = OracleRun(part, 0.1)
        out, lse = run.attention()
        keep = torch.from_numpy(np.concatenate([k.reshape(k.shape[0], -1) for k in run.keeps], 1))
        outs = [torch.zeros(1000, 4, 128, dtype=torch.float64) for _ in range(world)]
        keeps = [torch.zeros_like(keep) for _ in range(world)]
        dist.all_gather(outs, torch.from_numpy(out))
        dist.all_gather(keeps, keep)
        q.put((rank, part.workload.Hq, part.workload.Hkv,
               torch.cat(outs, 1).numpy() if rank == 0 else None,
               torch.cat(keeps, 0).numpy() if rank == 0 else None))
    finally:
        dist.destroy_process_group()


def test_head_split_gathers_to_the_whole_layer():
    """Two ranks, each running the path on its KV-head groups of one layer with no exchange:
    their gathered outputs and keep sets equal the whole layer's, computed in one process."""
    import dataclasses
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from block_sparse_long_qk_b200 import synthetic as S
    from _parity import OracleRun
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, 29513, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, Hq, Hkv, out, keep = q.get(timeout=300)
        res[r] = (Hq, Hkv, out, keep)
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert res[0][:2] == (4, 2) and res[1][:2] == (4, 2)
    w = dataclasses.replace(S.WORKLOADS["llama128k"], Hq=8, Hkv=4)
    full = OracleRun(S.make_inputs(w, seed=5, seqlens=(700, 300)), 0.1)
    ref, _ = full.attention()
    ref_keep = np.concatenate([k.reshape(k.shape[0], -1) for k in full.keeps], 1)
    assert np.array_equal(res[0][3], ref_keep)
    assert np.allclose(res[0][2], ref, rtol=0, atol=1e-12)

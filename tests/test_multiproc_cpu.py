"""The N > 1 bench path on CPU: two gloo ranks (127.0.0.1) exercise the
whole-job aggregation bench.py uses under torchrun -- units summed over the
replicas, time the slowest rank's -- and the reference arm's rank gating (only
rank 0 runs the oracle and prints)."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        res = {
            "max": bench.max_over_ranks(1.5 + rank, "cpu"),
            "sum": bench.sum_over_ranks(10.0 * (rank + 1), "cpu"),
            # rank 0 moved 100 units in 2 ms, rank 1 300 units in 4 ms
            "rate": bench.whole_job_rate([100.0, 300.0][rank], [2.0, 4.0][rank], "cpu"),
        }
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_whole_job_aggregation_over_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        with open(tmp_path / f"rank{r}.json") as f:
            res = json.load(f)
        assert res["max"] == 2.5
        assert res["sum"] == 30.0
        assert res["rate"] == pytest.approx(400.0 / 4e-3)


def test_single_process_aggregation_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.0, "cpu") == 3.0
    assert bench.whole_job_rate(50.0, 5.0, "cpu") == pytest.approx(10000.0)


def _reference_rank(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    import argparse
    import contextlib
    import io
    import bench
    import workloads as wl
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        args = argparse.Namespace(steps=1, warmup=1, seed=2, gpus=world)
        buf = io.StringIO()
        cfg = wl.small_variant(wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"], 2, 20, 40)
        with contextlib.redirect_stdout(buf):
            if rank != 0:
                bench.run_reference(args, cfg, rank, world)
        with open(os.path.join(out_dir, f"ref{rank}.txt"), "w") as f:
            f.write(buf.getvalue())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reference_arm_runs_on_rank_zero_only(tmp_path):
    port = _free_port()
    mp.start_processes(_reference_rank, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    assert (tmp_path / "ref1.txt").read_text() == ""      # rank 1 did no work, printed nothing


def _shard_rank(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    import bench
    import paged_kv_cache_338_b200 as pa
    import workloads as wl
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        cfg = wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"]
        mine = bench.sharded_cfg(cfg, 2, rank, world, pa)
        # every rank's share, gathered over the process group
        lens = torch.tensor(mine.fixed_lens, dtype=torch.int64)
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, torch.tensor([lens.numel()]))
        padded = torch.zeros(int(max(s.item() for s in sizes)), dtype=torch.int64)
        padded[:lens.numel()] = lens
        parts = [torch.zeros_like(padded) for _ in range(world)]
        dist.all_gather(parts, padded)
        got = sorted(sum((p[:int(n.item())].tolist() for p, n in zip(parts, sizes)), []))
        import dataclasses
        glob = dataclasses.replace(cfg, num_seqs=cfg.num_seqs * world)
        want = sorted(wl.draw_context_lens(glob, 2).tolist())
        with open(os.path.join(out_dir, f"shard{rank}.json"), "w") as f:
            json.dump({"n": lens.numel(), "tokens": int(lens.sum()), "union_ok": got == want,
                       "name": mine.name}, f)
    finally:
        dist.destroy_process_group()


def test_bench_splits_one_global_batch_by_sequence(tmp_path):
    """Under torchrun the decode bench splits one global batch (2 x 128
    sequences) over the ranks: the shares are disjoint, cover the batch, and
    carry about the same tokens."""
    port = _free_port()
    mp.start_processes(_shard_rank, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    res = [json.loads((tmp_path / f"shard{r}.json").read_text()) for r in range(2)]
    assert all(r["union_ok"] for r in res)
    assert res[0]["n"] + res[1]["n"] == 256
    assert abs(res[0]["tokens"] - res[1]["tokens"]) <= 8192
    assert res[0]["name"].endswith("shard0of2") and res[1]["name"].endswith("shard1of2")


def test_committed_traffic_needs_the_hash_of_the_current_kernels(tmp_path, monkeypatch):
    """A traffic record counts only when it was taken on the kernel sources
    that are built now: one without a hash, or with another one, gives None."""
    import bench
    import workloads as wl
    cfg = wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"]
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "csrc_sha256", lambda: "abc")
    f = tmp_path / "profiles" / f"traffic_{cfg.name}.json"
    rec = {"dram_bytes_per_launch": 123, "partition": 2048}
    f.write_text(json.dumps(rec))
    assert bench._traffic(cfg, 2048, False) is None
    f.write_text(json.dumps(dict(rec, csrc_sha256="def")))
    assert bench._traffic(cfg, 2048, False) is None
    f.write_text(json.dumps(dict(rec, csrc_sha256="abc")))
    assert bench._traffic(cfg, 2048, False) == 123
    assert bench._traffic(cfg, 512, False) is None          # taken for another partition

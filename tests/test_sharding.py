"""Token-range sharding across ranks (gloo, world size 2, CPU).

Each rank computes its shard with the CPU oracle using the shard's token
offset into the full-length position rows; rank 0 gathers the shards and checks
that they equal the unsharded result bit for bit.  This exercises the host
logic of the multi-GPU path (token ranges, offsets, gathering) without a GPU.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mrope_qk_norm_b200.sharding import shard_range


def test_shard_range_covers_exactly():
    for n in (0, 1, 7, 300, 8192, 8193):
        for world in (1, 2, 3, 8):
            spans = [shard_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import oracle
    import workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.config4(seed=7, T=301, Hq=4, Hkv=2)
        t0, t1 = shard_range(301, rank, world)
        s = w.streams[0]
        shard = W.StreamInputs(s.q[t0:t1], s.k[t0:t1], s.gamma_q, s.gamma_k)
        angle = W.AngleInputs(kind=w.angle.kind, section_mode=w.angle.section_mode,
                              sections=w.angle.sections, positions=w.angle.positions,
                              inv_freq=w.angle.inv_freq, token_offset=t0)
        q, k = oracle.qk_norm_rope([shard], w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, angle,
                                   norm=False)
        parts = [None] * world
        dist.all_gather_object(parts, (t0, t1, q, k))
        if rank == 0:
            full = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps,
                                       w.angle, norm=False)
            parts.sort(key=lambda x: x[0])
            ok = (np.array_equal(np.concatenate([p[2] for p in parts]), full[0]) and
                  np.array_equal(np.concatenate([p[3] for p in parts]), full[1]))
            with open(os.path.join(out_dir, "result"), "w") as f:
                f.write("ok" if ok else "mismatch")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_equal_unsharded(tmp_path):
    port = _free_port()
    mp.spawn(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    assert (tmp_path / "result").read_text() == "ok"


def _timing_worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mrope_qk_norm_b200.sharding import job_tokens_per_s, max_over_ranks
        local_ms = [30.0, 42.5][rank]          # the two ranks' own device times
        slowest = max_over_ranks(local_ms, dist, "cpu")
        value = job_tokens_per_s(world, 4608, slowest / 2000)
        with open(os.path.join(out_dir, "rank%d" % rank), "w") as f:
            f.write("%r %r" % (slowest, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_takes_the_slowest_rank(tmp_path):
    """bench.py's multi-rank aggregation: every rank gets the maximum of the
    ranks' device times, and whole-job throughput counts all ranks' tokens over
    that time (weak scaling)."""
    port = _free_port()
    mp.spawn(_timing_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        slowest, value = map(float, (tmp_path / ("rank%d" % r)).read_text().split())
        assert slowest == 42.5
        assert abs(value - 2 * 4608 / (42.5 / 2000 * 1e-3)) < 1e-6 * value

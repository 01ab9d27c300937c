"""The benchmark's multi-rank host logic on CPU (gloo, world size 2): rank
setup from the torchrun environment, barrier, max-over-ranks timing and the
whole-job aggregate -- without any GPU."""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup()
    try:
        assert (w, r, local) == (world, rank, rank)
        bench.barrier(w)
        # rank r "measured" 10 + r ms in total; every rank must see the max
        m = bench.max_over_ranks(10.0 + rank, w)
        tokens_per_step, steps = 512, 4
        value = tokens_per_step * w * steps / (m / 1e3)
        q.put((rank, m, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [m for _, m, _ in res] == [11.0, 11.0]
    assert all(abs(v - 512 * 2 * 4 / 0.011) < 1e-6 for _, _, v in res)


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    assert bench.dist_setup() == (1, 0, 0)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_algorithmic_work_figures():
    import bench
    # 1,288 B per token-head plus 64 KiB of final state per chain
    assert bench.prefill_bytes(1, 512, 16, False) == 512 * 16 * 1288 + 16 * 65536
    assert bench.prefill_bytes(1, 1, 1, True) == 1288 + 2 * 65536
    assert bench.prefill_flops(1, 1, 1) == 6 * 128 * 128 + 10 * 64 * 128 == 180224
    assert bench.decode_state_bytes(64, 16) == 134217728
    # per-channel gate: g is a vector of 128 fp32 per token-head
    assert bench.KDA_TOKEN_HEAD_BYTES == 3 * 256 + 512 + 4 + 512
    assert bench.kda_prefill_bytes(1, 512, 16, False) == 512 * 16 * 1796 + 16 * 65536
    # general head dims reduce to the 128 x 128 figures
    assert bench.prefill_bytes_dims(1, 512, 16, 128, 128, False) == bench.prefill_bytes(1, 512, 16, False)
    assert bench.prefill_flops_dims(1, 1, 1, 128, 128) == bench.prefill_flops(1, 1, 1)
    assert bench.prefill_bytes_dims(1, 1, 1, 64, 256, False) == 2 * 64 * 2 + 256 * 2 + 8 + 256 * 4 + 64 * 256 * 4

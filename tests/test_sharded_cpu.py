"""The N-split's bookkeeping on the CPU (gloo, world size 2 and 3): shard boundaries are
128-aligned and cover N, and the all-gather of the ranks' column blocks reassembles the
full output, with unequal shards (padded for the collective) and a ragged tail.  The
local products here are exact (integer-valued) float64 matmuls on the CPU standing in for
the GPU linear."""
import json
import os
import sys

import numpy as np
import pytest

from block_wise_w8a8_b200.sharded import BLOCK, shard_bounds

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N,world", [(4096, 2), (12288, 3), (16384, 8), (384, 2), (256, 3),
                                     (1000, 2), (128, 1), (0, 2)])
def test_shard_bounds(N, world):
    b = shard_bounds(N, world)
    assert len(b) == world and b[0][0] == 0 and b[-1][1] == N
    for (a0, a1), (c0, c1) in zip(b, b[1:]):
        assert a1 == c0
    widths = [n1 - n0 for n0, n1 in b]
    for n0, n1 in b:
        assert n0 % BLOCK == 0 and (n1 % BLOCK == 0 or n1 == N) and n1 >= n0
    full = [w for w in widths if w % BLOCK == 0]
    assert max(full, default=0) - min(full, default=0) <= BLOCK


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, M, K, N):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from block_wise_w8a8_b200.sharded import gather_columns, shard_bounds as sb
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r = np.random.default_rng(5)
        x = r.integers(-127, 128, (M, K)).astype(np.float64)     # integer products: exact
        w = r.integers(-127, 128, (N, K)).astype(np.float64)
        bounds = sb(N, world)
        n0, n1 = bounds[rank]
        y_local = torch.from_numpy(x @ w[n0:n1].T)
        y = gather_columns(y_local.contiguous(), bounds, rank)
        ok = bool(np.array_equal(y.numpy(), x @ w.T))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ok": ok, "shape": list(y.shape)}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,M,K,N", [(2, 256, 64, 512), (3, 128, 32, 640), (2, 128, 16, 1000)])
def test_gather_columns_gloo(tmp_path, world, M, K, N):
    import torch.multiprocessing as mp
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), M, K, N), nprocs=world, join=True)
    for rank in range(world):
        got = json.load(open(tmp_path / f"rank{rank}.json"))
        assert got["ok"] and got["shape"] == [M, N], (rank, got)

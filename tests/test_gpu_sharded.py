"""The N-split on one GPU: every rank's shard computed in turn (block-aligned rows of the
weight, the library's kernels) and placed at its columns equals the unsharded
w8a8_linear bit for bit, on the INT8 path and on the guard's BF16 path; and the
all-gather path end to end on a one-rank NCCL group."""
import datetime

import numpy as np
import pytest
import torch
import torch.distributed as dist

import block_wise_w8a8_b200 as w8
from block_wise_w8a8_b200.sharded import ShardedLinear
from gpu_util import dev_bf16, host_bits
from synth import f64_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert w8.device_error() == 0


def _case(M, K, N, seed):
    r = np.random.default_rng(seed)
    x = dev_bf16(f64_to_bf16_bits(r.standard_normal((M, K))))
    w = dev_bf16(f64_to_bf16_bits(r.standard_normal((N, K)) * K ** -0.5))
    b = dev_bf16(f64_to_bf16_bits(r.standard_normal(N) * 0.1))
    return x, w, b


@pytest.mark.parametrize("M,K,N,world", [(256, 512, 1024, 2), (384, 256, 1280, 3),
                                         (256, 384, 640, 8), (200, 256, 512, 2),
                                         (256, 256, 1000, 3)])
def test_shards_reassemble_the_unsharded_output(M, K, N, world):
    x, w, b = _case(M, K, N, M + K + N + world)
    y_ref, path = w8.linear(x, w8.W8A8Weight(w), b, return_path=True)
    y = torch.empty_like(y_ref)
    for rank in range(world):
        lin = ShardedLinear(w, b, rank, world)
        n0, n1 = lin.bounds[rank]
        y[:, n0:n1] = lin.local(x)
        assert lin.int8_path(M) == (path == w8.PATH_INT8)
    np.testing.assert_array_equal(host_bits(y), host_bits(y_ref))


def test_one_rank_nccl_gather():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        x, w, b = _case(512, 1024, 768, 9)
        y = ShardedLinear(w, b, 0, 1)(x)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host_bits(y), host_bits(w8.linear(x, w8.W8A8Weight(w), b)))
    finally:
        dist.destroy_process_group()

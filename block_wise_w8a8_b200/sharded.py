"""N-split of the guarded W8A8 linear over ranks: each rank holds a 128-aligned block of
the weight's output rows (W[n0:n1, :], with its INT8 codes and block scales), computes
Y[:, n0:n1] with the library's kernels, and one all-gather over the process group
(NCCL between GPUs) assembles Y[M, N] on every rank.

Block-aligned shards keep the method unchanged: a shard's codes and scales are the rows of
the whole weight's (each 128 x 128 block lies in one shard), and the guard is decided
once for the whole layer (M, K and N all multiples of 128, TurboT2VA paper, guard
paragraph), so every rank takes the path the unsharded call would take and the gathered
Y equals the unsharded output bit for bit.  The all-gather moves M x N x 2 bytes into
every rank; no kernel reads another GPU's memory.

The shard and gather bookkeeping (shard_bounds, gather_columns) is plain PyTorch and runs
on any process group, gloo on the CPU included."""
import torch
import torch.distributed as dist

BLOCK = 128


def shard_bounds(N, world):
    """[(n0, n1)] for ranks 0 .. world - 1: the ceil(N / 128) column blocks split as evenly
    as possible (the first N_blocks % world ranks get one more), every boundary a
    multiple of 128; the last shard ends at N (it holds a ragged tail when N % 128 != 0)."""
    if world <= 0 or N < 0:
        raise ValueError("world must be positive and N non-negative")
    nb = -(-N // BLOCK)
    base, extra = divmod(nb, world)
    bounds, b0 = [], 0
    for r in range(world):
        b1 = b0 + base + (1 if r < extra else 0)
        bounds.append((min(b0 * BLOCK, N), min(b1 * BLOCK, N)))
        b0 = b1
    return bounds


def gather_columns(y_local, bounds, rank, group=None, out=None):
    """All-gather the ranks' column blocks Y[:, n0_r:n1_r] (y_local is this rank's, [M, n1 -
    n0], contiguous) into out [M, N] on every rank.  Shards are padded to the widest one for
    the collective, which needs equal sizes."""
    world = len(bounds)
    M = y_local.shape[0]
    N = bounds[-1][1]
    n0, n1 = bounds[rank]
    if tuple(y_local.shape) != (M, n1 - n0):
        raise ValueError(f"rank {rank}: y_local must be [M, {n1 - n0}], got {tuple(y_local.shape)}")
    width = max(b - a for a, b in bounds)
    if out is None:
        out = torch.empty((M, N), dtype=y_local.dtype, device=y_local.device)
    if width == 0 or M == 0:
        return out
    send = y_local
    if n1 - n0 != width:
        send = torch.zeros((M, width), dtype=y_local.dtype, device=y_local.device)
        send[:, :n1 - n0] = y_local
    recv = torch.empty((world * M, width), dtype=y_local.dtype, device=y_local.device)
    dist.all_gather_into_tensor(recv, send.contiguous(), group=group)
    recv = recv.view(world, M, width)
    for r, (a, b) in enumerate(bounds):
        if b > a:
            out[:, a:b] = recv[r, :, :b - a]
    return out


class ShardedLinear:
    """This rank's part of an N-split W8A8 linear.  w_full: the layer's BF16 weight [N, K]
    (on this rank's device); bias: [N] or None.  The rank keeps W[n0:n1] (quantized once)
    and bias[n0:n1]."""

    def __init__(self, w_full, bias, rank, world, group=None):
        import block_wise_w8a8_b200 as w8
        self.N, self.K = w_full.shape
        self.rank, self.world, self.group = rank, world, group
        self.bounds = shard_bounds(self.N, world)
        n0, n1 = self.bounds[rank]
        self.w_bf16 = w_full[n0:n1].contiguous()
        self.weight = w8.W8A8Weight(self.w_bf16) if n1 > n0 else None
        self.bias = None if bias is None else bias[n0:n1].contiguous()

    def int8_path(self, M):
        """The guard, decided for the whole layer as the unsharded call decides it."""
        return M > 0 and M % BLOCK == 0 and self.K % BLOCK == 0 and self.N % BLOCK == 0 \
            and self.K <= 65536

    def local(self, x):
        """Y[:, n0:n1] on this rank: the INT8 path or the BF16 GEMM, as the guard says."""
        import block_wise_w8a8_b200 as w8
        n0, n1 = self.bounds[self.rank]
        M = x.shape[0]
        if n1 == n0:
            return torch.empty((M, 0), dtype=torch.bfloat16, device=x.device)
        if self.int8_path(M):
            y, path = w8.linear(x, self.weight, self.bias, return_path=True)
            if path != w8.PATH_INT8:
                raise RuntimeError("a shard left the INT8 path that the whole layer takes")
            return y
        return w8.bf16_linear(x, self.w_bf16, self.bias)

    def __call__(self, x, out=None):
        """Y = x W^T + bias [M, N] on every rank."""
        return gather_columns(self.local(x), self.bounds, self.rank, self.group, out)

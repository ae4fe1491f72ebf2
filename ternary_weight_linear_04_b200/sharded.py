"""BitLinear split by output features over the ranks of a process group.

Column-parallel (N-split): rank r holds rows [n0_r, n1_r) of W and the whole
activation row x; no reduction is needed, and the per-rank outputs are
gathered along N with one all-gather (NCCL over NVLink on GPUs).  gamma is
the mean |W| over the WHOLE matrix ([Production] "1. Absmean Weight
Quantization"): each rank forms the exact exponent-bucket sums of its rows,
an int64 sum all-reduce adds them (integer addition: the same totals for any
shard count or order), and every rank derives the identical gamma, so the
shards' codes and outputs are bit-identical to the single-GPU layer's.

The per-rank compute is the CUDA library (``bitlinear``); ``ops`` lets a
caller substitute another implementation of the same four calls.
"""
import torch
import torch.distributed as dist


def _after(stream, device):
    """torch's current stream (where collectives are ordered) waits for the
    library's work queued on `stream`."""
    if stream is not None:
        torch.cuda.current_stream(device).wait_stream(stream)


def _before(stream, device):
    """`stream` waits for what torch's current stream has queued (a
    collective's result)."""
    if stream is not None:
        stream.wait_stream(torch.cuda.current_stream(device))


def shard_bounds(N, world, rank):
    """Rows [n0, n1) of rank `rank`: contiguous, sizes differing by at most one
    (the first N % world ranks take one more)."""
    if not 0 <= rank < world:
        raise ValueError("rank %d outside a group of %d" % (rank, world))
    q, r = divmod(N, world)
    n0 = rank * q + min(rank, r)
    return n0, n0 + q + (1 if rank < r else 0)


class ShardedBitLinear:
    """One BitLinear layer (N x K) split by rows over `group`.

    W_shard: this rank's rows of the fp32 latent weights (n1 - n0 x K, on
    this rank's device); N: the whole matrix's out_features.
    """

    def __init__(self, W_shard, N, group=None, ops=None, stream=None):
        if ops is None:
            from . import bitlinear as ops
        self.ops = ops
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.N = N
        self.K = W_shard.shape[1]
        self.n0, self.n1 = shard_bounds(N, self.world, self.rank)
        if W_shard.shape[0] != self.n1 - self.n0:
            raise ValueError("rank %d holds %d rows; its shard is [%d, %d)"
                             % (self.rank, W_shard.shape[0], self.n0, self.n1))
        self.n_max = -(-N // self.world)
        self._bufs = {}
        if self.n1 > self.n0:
            buckets = ops.absmean_buckets(W_shard, stream=stream)
        else:  # more ranks than rows: this rank contributes nothing
            buckets = torch.zeros(256, dtype=torch.int64, device=W_shard.device)
        self._buckets = buckets  # kept: `stream` may still read it after __init__ returns
        _after(stream, W_shard.device)
        dist.all_reduce(buckets, op=dist.ReduceOp.SUM, group=group)
        _before(stream, W_shard.device)
        self.gamma = ops.gamma_from_buckets(buckets, N * self.K, stream=stream)
        self.packed = (ops.ternarise_pack(W_shard, self.gamma, stream=stream)
                       if self.n1 > self.n0 else None)

    def forward_local(self, x, out_dtype=torch.bfloat16, stream=None, out=None):
        """This rank's output columns: y[:, n0:n1] (M x (n1 - n0))."""
        n = self.n1 - self.n0
        if n == 0:
            return torch.empty((x.shape[0], 0), dtype=out_dtype, device=x.device)
        return self.ops.linear(x, self.packed, self.gamma, n, out_dtype=out_dtype,
                               weights_static=True, stream=stream, out=out)

    def _staging(self, M, dtype, device):
        """The send block and the gather buffer for M tokens of `dtype`,
        allocated on the first call with that shape and reused after it."""
        key = (M, dtype, device)
        bufs = self._bufs.get(key)
        if bufs is None:
            send = torch.empty(M * self.n_max, dtype=dtype, device=device)
            recv = torch.empty(self.world * M * self.n_max, dtype=dtype, device=device)
            bufs = self._bufs[key] = (send, recv)
        return bufs

    def forward(self, x, out_dtype=torch.bfloat16, stream=None, out=None):
        """The whole output y (M x N) on every rank: local columns, then one
        all-gather of equal-sized (padded) per-rank blocks along N.  The layer
        writes its columns straight into the send block when they are
        contiguous there (one token, or an even split); with one token and an
        even split the gather lands directly in y.  The send block and the
        gather buffer are kept between calls (per token count and dtype), so
        a call allocates nothing but y itself, and not that when `out` (a
        contiguous M x N tensor) is given."""
        M = x.shape[0]
        n = self.n1 - self.n0
        if out is None:
            out = torch.empty((M, self.N), dtype=out_dtype, device=x.device)
        send, recv = self._staging(M, out_dtype, x.device)
        if n > 0 and (M == 1 or n == self.n_max):
            self.forward_local(x, out_dtype, stream, out=send[:M * n].view(M, n))
            _after(stream, x.device)
        elif n > 0:
            y_local = self.forward_local(x, out_dtype, stream)
            _after(stream, x.device)
            send.view(M, self.n_max)[:, :n] = y_local
        if self.n_max * self.world == self.N and M == 1 and out.is_contiguous():
            # rank-major blocks are already y's layout
            dist.all_gather_into_tensor(out.view(-1), send, group=self.group)
            return out
        dist.all_gather_into_tensor(recv, send, group=self.group)
        blocks = recv.view(self.world, M, self.n_max)
        parts = []
        for r in range(self.world):
            a, b = shard_bounds(self.N, self.world, r)
            parts.append(blocks[r, :, :b - a])
        return torch.cat(parts, dim=1, out=out)

"""N-split (column-parallel) layer over a process group, on CPU.

Runs gloo ranks on 127.0.0.1 with a CPU stand-in for the four per-rank
library calls (exact integer bucket sums and the oracle), and checks the
host logic the GPU build shares: the row split, the int64 all-reduce of the
exponent buckets (gamma of the WHOLE matrix on every rank, [Production]
"1. Absmean Weight Quantization"), each shard's codes, and the all-gather
that assembles y.  Expected values come from the oracle on the unsplit
matrix.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleOps:
    """The per-rank calls on CPU tensors: bucket sums as exact integers,
    gamma from them with Python's correctly rounded division, codes and the
    layer from the oracle."""

    @staticmethod
    def absmean_buckets(W, stream=None):
        u = np.abs(W.numpy()).view(np.uint32).ravel()
        e = (u >> 23) & 0xFF
        m = np.where(e > 0, (u & 0x7FFFFF) | 0x800000, u & 0x7FFFFF).astype(np.int64)
        b = np.where(e > 0, e, 1)
        out = np.zeros(256, np.int64)
        for v in np.unique(b):
            out[v] = int(m[b == v].sum())
        return torch.from_numpy(out)

    @staticmethod
    def gamma_from_buckets(buckets, count, stream=None):
        num = sum(int(v) << (b - 1) for b, v in enumerate(buckets.tolist()) if 1 <= b <= 254)
        S = num / (1 << 149)  # the exact sum rounded once to fp64
        g = max(np.float32(S / count), np.float32(1e-5))
        return torch.tensor([g], dtype=torch.float32)

    @staticmethod
    def ternarise_pack(W, gamma, stream=None):
        from oracle import reference as ref
        return torch.from_numpy(ref.pack2(ref.ternarise(W.numpy(), np.float32(gamma.item()))))

    @staticmethod
    def linear(x, packed, gamma, N, out_dtype=torch.bfloat16, weights_static=False, stream=None,
               out=None):
        from oracle import reference as ref
        xq, eta, _ = ref.quant_act(x.float().numpy())
        _, y = ref.forward(xq, eta, packed.numpy(), np.float32(gamma.item()), x.shape[1])
        yt = torch.from_numpy(np.ascontiguousarray(y)).to(out_dtype)
        assert yt.shape == (x.shape[0], N)
        if out is not None:
            out.copy_(yt)
            return out
        return yt


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, N, K, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta
    from oracle import reference as ref
    from ternary_weight_linear_04_b200 import inputs
    from ternary_weight_linear_04_b200.sharded import ShardedBitLinear, shard_bounds
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world, timeout=timedelta(seconds=60))
    try:
        W, x = inputs.make_case(900 + N + K, 3, K, N, act_dtype="bf16")
        n0, n1 = shard_bounds(N, world, rank)
        layer = ShardedBitLinear(torch.from_numpy(W[n0:n1].copy()), N, ops=OracleOps)
        g_ref, _ = ref.absmean_gamma(W)
        packed_ref = ref.pack2(ref.ternarise(W, g_ref))
        xq, eta, _ = ref.quant_act(x)
        _, y_ref = ref.forward(xq, eta, packed_ref, g_ref, K)
        res = {"gamma": bool(layer.gamma.numpy().view(np.uint32)[0] == np.float32(g_ref).view(np.uint32)),
               "packed": layer.packed is None or bool(np.array_equal(layer.packed.numpy(), packed_ref[n0:n1]))}
        for M in (1, 3):
            xt = torch.from_numpy(x[:M]).to(torch.bfloat16)
            want = torch.from_numpy(np.ascontiguousarray(y_ref[:M])).to(torch.bfloat16)
            y = layer.forward(xt)
            res["y%d" % M] = bool(y.shape == (M, N) and torch.equal(y.view(torch.int16),
                                                                    want.view(torch.int16)))
            loc = layer.forward_local(xt)
            res["local%d" % M] = bool(torch.equal(loc.view(torch.int16),
                                                  want[:, n0:n1].contiguous().view(torch.int16)))
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N,K", [(2, 389, 200), (2, 390, 64), (3, 7, 33), (3, 2, 40)])
def test_n_split_matches_the_unsplit_layer(world, N, K):
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, N, K, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    got = dict(q.get() for _ in range(world))
    for r in range(world):
        assert all(got[r].values()), (r, got[r])


def test_shard_bounds_cover_the_rows_once():
    sys.path.insert(0, ROOT)
    from ternary_weight_linear_04_b200.sharded import shard_bounds
    for N in (1, 2, 7, 8, 389, 8640):
        for world in (1, 2, 3, 4, 8):
            b = [shard_bounds(N, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == N
            assert all(b[i][1] == b[i + 1][0] for i in range(world - 1))
            sizes = [n1 - n0 for n0, n1 in b]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        shard_bounds(8, 2, 2)


def test_bucket_stand_in_reproduces_the_oracle_gamma():
    """The CPU stand-in's bucket sums, split any way and added as int64,
    give the oracle's whole-matrix gamma bit for bit."""
    sys.path.insert(0, ROOT)
    from oracle import reference as ref
    rng = np.random.default_rng(2)
    for scale in (0.02, 1e-30, 3e30):
        W = (rng.standard_normal((37, 53)) * scale).astype(np.float32)
        W[0, :5] = np.float32(1e-42)  # subnormals
        g_ref, _ = ref.absmean_gamma(W)
        for cut in (0, 1, 20, 36):
            parts = [W[:cut], W[cut:]]
            tot = sum(OracleOps.absmean_buckets(torch.from_numpy(p.copy())) for p in parts if len(p))
            g = OracleOps.gamma_from_buckets(tot, W.size)
            assert g.numpy().view(np.uint32)[0] == np.float32(g_ref).view(np.uint32)

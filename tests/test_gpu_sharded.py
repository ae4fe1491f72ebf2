"""Split packing steps and the N-split layer on the GPU.

[Production] "1. Absmean Weight Quantization": gamma is the mean over the
whole matrix, so row shards packed separately must reproduce the unsplit
matrix's gamma and codes bit for bit.  One GPU emulates the shards (bucket
sums added as int64, as the all-reduce does); a one-rank NCCL group runs the
sharded layer's collectives.
"""
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch

from oracle import native as orc
from ternary_weight_linear_04_b200 import bitlinear as bl
from ternary_weight_linear_04_b200 import build as libbuild
from ternary_weight_linear_04_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    assert bl.device_error() == 0


@pytest.mark.parametrize("N,K,cuts", [(389, 1600, (0, 1, 200, 388)), (64, 3200, (17, 40)),
                                      (5, 7, (2,))])
def test_split_packing_equals_whole_matrix(N, K, cuts):
    W, _ = inputs.make_case(4400 + N + K, 1, K, N)
    Wd = torch.from_numpy(W).cuda()
    packed, gamma = bl.pack_weights(Wd)
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    assert gamma.cpu().numpy().view(np.uint32)[0] == np.float32(ref_gamma).view(np.uint32)
    bounds = [0, *cuts, N]
    shards = [(a, b) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]
    tot = torch.zeros(256, dtype=torch.int64, device="cuda")
    for a, b in shards:
        tot += bl.absmean_buckets(Wd[a:b].contiguous())
    g = bl.gamma_from_buckets(tot, N * K)
    assert g.cpu().numpy().view(np.uint32)[0] == gamma.cpu().numpy().view(np.uint32)[0]
    parts = [bl.ternarise_pack(Wd[a:b].contiguous(), g) for a, b in shards]
    np.testing.assert_array_equal(torch.cat(parts).cpu().numpy(), ref_packed)
    # the whole matrix through the steps equals pack_weights
    whole = bl.ternarise_pack(Wd, bl.gamma_from_buckets(bl.absmean_buckets(Wd), N * K))
    np.testing.assert_array_equal(whole.cpu().numpy(), packed.cpu().numpy())


def test_sharded_layer_on_a_one_rank_nccl_group():
    import torch.distributed as dist
    from ternary_weight_linear_04_b200.sharded import ShardedBitLinear
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0,
                            world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        N, K = 389, 1600
        W, x = inputs.make_case(4500, 4, K, N, act_dtype="bf16")
        Wd = torch.from_numpy(W).cuda()
        packed, gamma = bl.pack_weights(Wd)
        stream = torch.cuda.Stream()
        layer = ShardedBitLinear(Wd, N, stream=stream)
        torch.cuda.synchronize()
        assert torch.equal(layer.gamma, gamma) and torch.equal(layer.packed, packed)
        xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
        for M in (1, 4):
            want = bl.linear(xd[:M], packed, gamma, N)
            got = layer.forward(xd[:M], stream=stream)
            torch.cuda.synchronize()
            assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    finally:
        dist.destroy_process_group()

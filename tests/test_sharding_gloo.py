"""Multi-rank host logic on CPU (gloo, world size 2): the block partition and the
8-byte (-delta, Delta) exchange between the two halves of a sharded step.

Each rank takes its shard of a vector, computes the shard's residual min/max
at t = 1 with the oracle (blocks are independent at t = 1), writes the pair
into a header the way the select kernel does and runs the product's
all-reduce; every rank must then hold the oracle's (delta_2, Delta_2) of the
whole vector."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from compressed_state_optimizer_b200 import sharding

D, BD, KB = 7 * 512 + 77, 512, 6


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _grads():
    import pins
    return pins.normal_bf16(D, 2024, scale=0.5)


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b0, nb = sharding.shard_blocks(D, BD, rank, world)
        lo, hi = b0 * BD, min(D, (b0 + nb) * BD)
        g = _grads()[lo:hi].copy()
        st = oracle.new_state(hi - lo, BD, KB, 2)
        p = np.zeros(hi - lo, dtype=np.float32)
        oracle.step(st, p, g, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.0, t=1, seed=3)
        header = torch.zeros(256, dtype=torch.uint8)
        header[8:16] = torch.from_numpy(sharding.pack_pair(st.scal[0], st.scal[1]).view(np.uint8))
        sharding.combine_minmax_(header, 8)
        out[rank] = sharding.unpack_pair(header[8:16].view(torch.int32).numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_minmax_exchange_matches_whole_vector(oracle_lib, world):
    import oracle
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    st = oracle.new_state(D, BD, KB, 2)
    p = np.zeros(D, dtype=np.float32)
    oracle.step(st, p, _grads(), lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.0, t=1, seed=3)
    for r in range(world):
        assert out[r] == (float(st.scal[0]), float(st.scal[1]))


def test_shard_blocks_partition():
    for d, bd, world in [(10 * 64 + 1, 64, 3), (411281 * 16384 - 12288, 16384, 8), (5, 2, 3)]:
        nb = -(-d // bd)
        cover = []
        for r in range(world):
            b0, n = sharding.shard_blocks(d, bd, r, world)
            assert n >= 1
            cover.extend(range(b0, b0 + n))
        assert cover == list(range(nb))
    with pytest.raises(ValueError):
        sharding.shard_blocks(3 * 64, 64, 0, 4)


def test_pair_encoding_orders_like_values():
    rng = np.random.default_rng(0)
    for _ in range(1000):
        a, b = sorted(np.abs(rng.standard_normal(2) * 10.0 ** rng.integers(-30, 30, 2)))
        pa, pb = sharding.pack_pair(-a, a), sharding.pack_pair(-b, b)
        assert pa[0] <= pb[0] and pa[1] <= pb[1]
    assert tuple(sharding.pack_pair(-0.0, -0.0)) == (0, 0)

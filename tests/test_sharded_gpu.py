"""The sharded step on one GPU: two shard handles of one vector, run one after
the other with the 8-byte (-delta, Delta) exchange done as a device-side MAX
(what the all-reduce of a 2-rank run computes), must reproduce the unsharded
step bit for bit: codes, window, scalars and parameters. No kernel waits on
another; each launch completes on its own."""
import pytest

from conftest import cuda_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("world", [2, 3])
def test_shards_reproduce_whole_vector(world):
    import torch
    from compressed_state_optimizer_b200 import MicroAdam, sharding, workloads
    d, Bd, kb, m = 7 * 16384 + 5000, 16384, 164, 4
    w = workloads.Workload("shards", d, Bd, kb, m, "t3", 8)
    hyper = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.0, seed=77)
    whole = MicroAdam(d, block_size=Bd, k_per_block=kb, window=m)
    shards = [MicroAdam(d, block_size=Bd, k_per_block=kb, window=m,
                        shard=sharding.shard_blocks(d, Bd, r, world)) for r in range(world)]
    p0 = workloads.make_params(d).cuda()
    p_whole = p0.clone()
    p_sh = [p0[s.offset: s.offset + s.d].clone() for s in shards]
    st_whole = whole.new_state()
    st_sh = [s.new_state() for s in shards]
    for t in range(1, 9):
        g = workloads.make_grads(w, t).cuda()
        whole.step(p_whole, g, st_whole, t=t, **hyper)
        g_sh = [g[s.offset: s.offset + s.d] for s in shards]
        for s, p, gs, st in zip(shards, p_sh, g_sh, st_sh):
            s.select(p, gs, st, t=t, **hyper)
        o = shards[0].minmax_offset(t)
        pair = st_sh[0][o:o + 8].view(torch.int32).clone()
        for st in st_sh[1:]:
            pair = torch.maximum(pair, st[o:o + 8].view(torch.int32))
        for st in st_sh:
            st[o:o + 8].view(torch.int32).copy_(pair)
        for s, p, gs, st in zip(shards, p_sh, g_sh, st_sh):
            s.apply(p, gs, st, t=t, **hyper)
    torch.cuda.synchronize()
    lw = whole.layout
    codes = torch.cat([st[s.layout.codes: s.layout.codes + s.d // 2 + (s.d % 2)]
                       for s, st in zip(shards, st_sh)])
    assert torch.equal(codes, st_whole[lw.codes: lw.codes + (d + 1) // 2])
    win = torch.cat([st[s.layout.window: s.layout.bytes] for s, st in zip(shards, st_sh)])
    assert torch.equal(win, st_whole[lw.window: lw.bytes])
    for st in st_sh:
        assert torch.equal(st[:16], st_whole[:16])
    assert torch.equal(torch.cat(p_sh), p_whole)

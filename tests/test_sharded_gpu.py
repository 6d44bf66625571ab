"""The sharded step on one GPU: shard handles of one vector, run one after the
other with the 8-byte (-delta, Delta) exchange done as a device-side MAX (what
the all-reduce of a multi-rank run computes), against the oracle run on the
whole vector, every step: the shards' codes, window rows (as sets of pairs)
and scalars bit for bit, their parameters within 1e-5; and bit for bit against
the unsharded step (window rows as sets of pairs). No kernel waits on another;
each launch completes on its own."""
import numpy as np
import pytest

import oracle
import state_view
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
    ost = oracle.new_state(d, Bd, kb, m)
    p_ref = p0.cpu().numpy().copy()
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
        oracle.step(ost, p_ref, workloads.bf16_bits(g), t=t, **hyper)
        torch.cuda.synchronize()
        # the shards, reassembled in the whole vector's layout, against the oracle
        lw = whole.layout
        sb = st_sh[0][:lw.codes].cpu().numpy().copy()
        codes = torch.cat([st[s.layout.codes: s.layout.codes + s.d // 2 + (s.d % 2)]
                           for s, st in zip(shards, st_sh)]).cpu().numpy()
        win = torch.cat([st[s.layout.window: s.layout.bytes]
                         for s, st in zip(shards, st_sh)]).cpu().numpy()
        assert np.array_equal(codes, ost.codes), t
        lo, hi = state_view.header_scalars(sb, t + 1)
        assert np.float32(lo) == ost.scal[0] and np.float32(hi) == ost.scal[1], t
        kp = lw.row_stride
        wv = win.view(np.uint32).reshape(lw.blocks, m, kp)[:, :, :kb].transpose(1, 0, 2)
        for s_ in range(max(1, t - m + 1), t + 1):
            r = s_ % m
            gi, gv = state_view.canonical_words(wv[r])
            assert np.array_equal(gi, ost.G_idx[r]), (t, s_)
            assert np.array_equal(gv, ost.G_val[r]), (t, s_)
        p = torch.cat(p_sh).cpu().numpy().astype(np.float64)
        tol = 1e-5 * np.maximum(np.abs(p_ref.astype(np.float64)), hyper["lr"])
        assert np.all(np.abs(p - p_ref) <= tol), t
    torch.cuda.synchronize()
    codes = torch.cat([st[s.layout.codes: s.layout.codes + s.d // 2 + (s.d % 2)]
                       for s, st in zip(shards, st_sh)])
    assert torch.equal(codes, st_whole[lw.codes: lw.codes + (d + 1) // 2])
    win = torch.cat([st[s.layout.window: s.layout.bytes] for s, st in zip(shards, st_sh)])
    # the whole vector takes the fused step, which lists a row in another order
    wi, wv = state_view.canonical_words(win.cpu().numpy().view(np.uint32).reshape(-1, lw.row_stride))
    ri, rv = state_view.canonical_words(
        st_whole[lw.window: lw.bytes].cpu().numpy().view(np.uint32).reshape(-1, lw.row_stride))
    assert np.array_equal(wi, ri) and np.array_equal(wv, rv)
    for st in st_sh:
        assert torch.equal(st[:16], st_whole[:16])
    assert torch.equal(torch.cat(p_sh), p_whole)

"""The multi-GPU Ring Attention driver's host logic on CPU ranks (gloo,
127.0.0.1): real send/receive of key/value blocks between 2 and 4 ranks, the
block each rank holds at each step, and the merged result against the
single-process attention of the whole sequence.

The per-block attention and its merge are the float64 oracle here (the
driver takes them as an argument); on GPUs ring_attention_dist binds them to
librcx kernels and NCCL."""

import math
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

B, Hq, Hkv, D = 1, 4, 2, 16


def _inputs(N):
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B, N, Hq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, N, Hkv, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, N, Hkv, D, generator=g, dtype=torch.float64)
    return q, k, v


def _worker(rank, world, port, N, window, n_sink, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from oracle import rcx_oracle as orc
    from rope_context_extension_scaled_b200 import ring_dist
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        shard = N // world
        q, k, v = _inputs(N)
        inv, t = orc.rope_freqs(orc.NTK, 1e4, D, 64, 256)
        scale = 1.0 / (math.sqrt(D) * t)
        lo, hi = rank * shard, (rank + 1) * shard
        qs = q[:, lo:hi].clone()
        # this rank's key shard, rotated once at its global positions
        ks = torch.from_numpy(orc.rope_rotate(k[0, lo:hi].numpy(), np.arange(lo, hi), inv))[None]
        kv_bufs = [(ks.clone(), v[:, lo:hi].clone()), (torch.empty_like(ks), torch.empty_like(ks))]
        held = []

        def attend(qq, kb, vb, o, l, q_start, k_start, prev):
            # the block held must be the global block starting at k_start
            b = k_start // shard
            exp_k = orc.rope_rotate(k[0, k_start:k_start + shard].numpy(), np.arange(k_start, k_start + shard), inv)
            held.append((b, bool(np.array_equal(kb[0].numpy(), exp_k)),
                         bool(torch.equal(vb, v[:, k_start:k_start + shard]))))
            qr = orc.rope_rotate(qq[0].numpy(), np.arange(q_start, q_start + shard), inv)
            O, L = orc.attention(qr, kb[0].numpy(), vb[0].numpy(), scale, window=window, n_sink=n_sink,
                                 q_index=np.arange(q_start, q_start + shard),
                                 k_index=np.arange(k_start, k_start + shard))
            if prev is not None:   # LSE merge with the partial over earlier blocks
                O, L = orc.merge(prev[0][0].numpy().transpose(1, 0, 2), prev[1][0].numpy(),
                                 O.transpose(1, 0, 2), L)
                O = O.transpose(1, 0, 2)
            o[0] = torch.from_numpy(np.ascontiguousarray(O))
            l[0] = torch.from_numpy(np.ascontiguousarray(L))

        out = torch.empty_like(qs)
        lse = torch.empty(B, Hq, shard, dtype=torch.float64)
        acc, lacc = torch.empty_like(qs), torch.empty_like(lse)
        exch = ring_dist.Exchange() if world > 1 else None
        ring_dist.ring_forward(qs, kv_bufs, rank=rank, world=world, window=window, n_sink=n_sink,
                               attend=attend, exchange=exch, out=out, lse=lse, acc=acc, lacc=lacc)
        # the whole sequence in one process
        qr = orc.rope_rotate(q[0].numpy(), np.arange(N), inv)
        kr = orc.rope_rotate(k[0].numpy(), np.arange(N), inv)
        O, L = orc.attention(qr, kr, v[0].numpy(), scale, window=window, n_sink=n_sink)
        sched = [(s.t, s.block, s.visible) for s in ring_dist.ring_schedule(rank, world, shard, window, n_sink)]
        out_q.put((rank, held, sched, float(np.abs(out[0].numpy() - O[lo:hi]).max()),
                   bool(np.array_equal(np.isneginf(lse[0].numpy()), np.isneginf(L[:, lo:hi]))),
                   float(np.nan_to_num(np.abs(lse[0].numpy() - L[:, lo:hi]), posinf=0.0).max())))
    finally:
        dist.destroy_process_group()


def _run(world, port, N, window=0, n_sink=0):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, N, window, n_sink, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    return sorted(res)


@pytest.mark.parametrize("world,window,n_sink", [(2, 0, 0), (4, 0, 0), (4, 20, 3)])
def test_ring_exchange_and_merge_on_gloo_ranks(world, window, n_sink):
    N = 32 * world
    res = _run(world, 29541 + world + window, N, window, n_sink)
    shard = N // world
    for rank, held, sched, o_err, inf_ok, l_err in res:
        # step t holds block (rank - t) mod P; blocks after the shard are skipped (causal)
        assert [b for _, b, _ in sched] == [(rank - t) % world for t in range(world)]
        vis_blocks = [b for _, b, vis in sched if vis]
        assert all(b <= rank for b in vis_blocks)
        # every visible step attended to the right block, received over the ring
        assert [h[0] for h in held] == vis_blocks
        assert all(kok and vok for _, kok, vok in held)
        assert inf_ok and o_err < 1e-12 and l_err < 1e-12, (rank, o_err, l_err)
    if window:
        # with a window of 20 keys + 3 sinks, rank 3 sees block 0 (sinks) but not block 1
        r3 = [s for s in res if s[0] == 3][0]
        assert [(b, v) for _, b, v in r3[2]] == [(3, True), (2, True), (1, False), (0, True)]


def test_ring_schedule_single_rank_and_block_visibility():
    sys.path.insert(0, ROOT)
    from rope_context_extension_scaled_b200 import ring_dist
    s = ring_dist.ring_schedule(0, 1, 100)
    assert len(s) == 1 and s[0].block == 0 and s[0].visible and s[0].first and s[0].last
    # 16-way ring of the 1M workload: rank r sees r + 1 blocks, last one on step r
    for r in (0, 5, 15):
        s = ring_dist.ring_schedule(r, 16, 65536)
        vis = [x.t for x in s if x.visible]
        assert vis == list(range(r + 1)) and s[0].first and s[r].last
    assert ring_dist.block_visible(100, 199, 0, 49, 50, 4)          # sinks
    assert not ring_dist.block_visible(100, 199, 10, 49, 50, 4)     # outside window, no sinks
    assert not ring_dist.block_visible(0, 99, 100, 199, 0, 0)       # after every query

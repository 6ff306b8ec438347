"""The multi-GPU Ring Attention driver bound to librcx kernels, on one GPU:
each rank's loop runs in turn in this process, with a stand-in exchange that
hands it the block the ring would deliver at each step (the global block
(rank - t - 1) mod P, rotated at its global positions).  The exchange itself
is covered by the gloo tests; this checks the per-rank compute path (key shard
rotation at global positions, per-block attention with q_start / k_start,
LSE merges in the attention epilogue) against the float64 oracle on the
whole sequence."""

import numpy as np
import pytest
import torch

from rope_context_extension_scaled_b200 import _lib, ring_dist
from rope_context_extension_scaled_b200.inputs import make_qkv
from tests._parity import all_rows, assert_bf16, assert_f32, errors, gather_gpu, oracle_rows, schedule

pytestmark = pytest.mark.gpu


class BlockFeed:
    """Exchange stand-in: the receive buffers get the block the ring would bring."""

    def __init__(self, rank, world, k_rot, v, shard):
        self.rank, self.world, self.k_rot, self.v, self.shard, self.t = rank, world, k_rot, v, shard, 0

    def post(self, send, recv):
        b = (self.rank - self.t - 1) % self.world
        sl = slice(b * self.shard, (b + 1) * self.shard)
        recv[0].copy_(self.k_rot[:, sl])
        recv[1].copy_(self.v[:, sl])
        self.t += 1
        return []


@pytest.mark.parametrize("dtype,d,world,window,n_sink", [
    (torch.bfloat16, 128, 4, 0, 0), (torch.bfloat16, 128, 2, 0, 0), (torch.bfloat16, 128, 4, 300, 4),
    (torch.float32, 64, 4, 0, 0)])
def test_ring_dist_per_rank_path_matches_oracle(dtype, d, world, window, n_sink):
    N = 1024
    shard = N // world
    q, k, v = make_qkv(1, N, 4, 2, d, dtype, seed=40, device="cuda")
    inv, t, oinv, ot = schedule(_lib.NTK, 5e5, d, 256, 2048)
    k_rot = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, k_out=k_rot)
    attend = ring_dist.librcx_attend(inv, t, window, n_sink)
    o = torch.empty_like(q)
    lse = torch.empty(1, 4, N, dtype=torch.float32, device="cuda")
    for r in range(world):
        sl = slice(r * shard, (r + 1) * shard)
        qs = q[:, sl].contiguous()
        kv_bufs, acc, lacc = ring_dist.ring_buffers(qs, k[:, sl].contiguous(), v[:, sl].contiguous(), inv,
                                                    r * shard)
        out = torch.empty_like(qs)
        ls = torch.empty(1, 4, shard, dtype=torch.float32, device="cuda")
        ring_dist.ring_forward(qs, kv_bufs, rank=r, world=world, window=window, n_sink=n_sink, attend=attend,
                               exchange=BlockFeed(r, world, k_rot, v, shard), out=out, lse=ls, acc=acc, lacc=lacc)
        o[:, sl] = out
        lse[:, :, sl] = ls
    torch.cuda.synchronize()
    rows = all_rows(N, 4)
    Or, Lr = oracle_rows(q[0], k[0], v[0], oinv, ot, rows, window, n_sink)
    err = errors(*gather_gpu(o, lse, rows), Or, Lr)
    print(err)
    (assert_bf16 if dtype == torch.bfloat16 else assert_f32)(err)

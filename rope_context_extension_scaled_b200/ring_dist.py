"""Ring Attention across GPUs: one sequence shard per rank, KV blocks passed
around the ring.

"Context window extension: 4K to 1M" section 5.3 gives the loop: each rank
keeps its query shard, computes attention against the key/value block it
currently holds, sends that block to rank + 1 and receives the next one from
rank - 1; section 5.4 (Flash Ring Attention) runs the blockwise kernel on each
step.  The kwkr.cn long-context article, section 2.2, states the same roll of
the KV chunks by one position with the partial results aggregated online.

Layout.  The global sequence of N tokens is cut into P = world-size
contiguous shards of Ns = N / P tokens; rank r holds query, key and value rows
[r Ns, (r + 1) Ns) of every head.  At step t rank r holds KV block (r - t) mod P
(its own block at t = 0).  Positions are global token indices: the query shard
is rotated in the attention kernel's tile load at q_start = r Ns, and the key
shard is rotated once, before the ring starts, at positions r Ns .. (r+1) Ns - 1,
so the blocks that travel are already rotated.

Per step the exchange of the next block (send to r + 1, receive from r - 1, one
batched point-to-point call) is posted before the step's attention is launched,
so with NCCL the transfer over NVLink runs on NCCL's stream while the kernel
runs on the compute stream.  Received blocks land in a local double buffer in
this GPU's HBM; the attention kernel's TMA loads only ever read local memory.

Causal masking makes blocks b > r invisible to rank r: those steps launch
nothing but still forward the block.  Partial results merge by the LSE rule
("output += block_output" of section 5.3 made exact): the first visible block
writes the fp32 accumulator, later blocks are merged into it in the
attention kernel's epilogue, and the last step writes the output in its final
dtype.

The driver is plain host logic; the per-block attention (with its merge) and
the exchange are passed in.  ``ring_attention_dist`` binds them to librcx
kernels and torch.distributed (NCCL on GPUs); it fails if the CUDA library is
missing.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence

import torch


@dataclass(frozen=True)
class RingStep:
    t: int              # ring step
    block: int          # KV block held at this step: (rank - t) mod P
    visible: bool       # does any (query, key) pair of this shard and block pass the mask?
    first: bool         # first visible block of this rank (writes the accumulator)
    last: bool          # last visible block of this rank (writes the final output)


def block_visible(i0: int, i1: int, j0: int, j1: int, window: int, n_sink: int) -> bool:
    """Does any query i in [i0, i1] see any key j in [j0, j1]?  Causal mask
    with a sliding window of ``window`` keys (0 = none) and ``n_sink`` sink
    keys ("Context window extension: 4K to 1M" 4.1, 4.2)."""
    if j0 > i1:
        return False
    if window == 0:
        return True
    if j1 > i0 - window:
        return True
    return j0 < n_sink


def ring_schedule(rank: int, world: int, shard: int, window: int = 0, n_sink: int = 0) -> List[RingStep]:
    """The steps rank ``rank`` takes in a ring of ``world`` ranks with shards
    of ``shard`` tokens: at step t it holds block (rank - t) mod world."""
    i0, i1 = rank * shard, (rank + 1) * shard - 1
    steps = []
    for t in range(world):
        b = (rank - t) % world
        vis = block_visible(i0, i1, b * shard, (b + 1) * shard - 1, window, n_sink)
        steps.append([t, b, vis])
    vis_t = [s[0] for s in steps if s[2]]
    first = vis_t[0] if vis_t else -1
    last = vis_t[-1] if vis_t else -1
    return [RingStep(t, b, v, t == first, t == last) for t, b, v in steps]


class Exchange:
    """One ring hop: send tensors to rank + 1 and receive the same shapes
    from rank - 1, as one batched point-to-point call of torch.distributed."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def _global(self, r):
        return r if self.group is None else self.dist.get_global_rank(self.group, r)

    def post(self, send: Sequence[torch.Tensor], recv: Sequence[torch.Tensor]):
        dist = self.dist
        nxt = self._global((self.rank + 1) % self.world)
        prv = self._global((self.rank - 1) % self.world)
        ops = [dist.P2POp(dist.isend, x, nxt, self.group) for x in send]
        ops += [dist.P2POp(dist.irecv, x, prv, self.group) for x in recv]
        return dist.batch_isend_irecv(ops)


def ring_forward(q: torch.Tensor, kv_bufs: Sequence[Sequence[torch.Tensor]], *, rank: int, world: int,
                 window: int, n_sink: int, attend: Callable, exchange: Optional[Exchange],
                 out: torch.Tensor, lse: Optional[torch.Tensor], acc: torch.Tensor, lacc: torch.Tensor):
    """Host loop of the ring on one rank.

    q: this rank's query shard [B, Ns, Hq, d] (raw; rotated by ``attend``).
    kv_bufs: two (k, v) buffer pairs of the block shape [B, Ns, Hkv, d];
    kv_bufs[0] starts out holding this rank's own block (keys already
    rotated): step 0 attends to it and sends it on.  The buffers are
    overwritten by the blocks received.
    attend(q, k, v, o, l, q_start, k_start, prev): attention of the shard
    against one block into o and l (fp32 LSE); prev is None, or the
    (o_prev, l_prev) partial over earlier blocks, which attend merges in by the
    LSE rule (o, l may be o_prev, l_prev).
    acc, lacc: fp32 accumulator [B, Ns, Hq, d] and its LSE [B, Hq, Ns].
    exchange: an Exchange, or None for a single rank.
    Returns (out, lse)."""
    shard = q.shape[1]
    steps = ring_schedule(rank, world, shard, window, n_sink)
    n_vis = sum(s.visible for s in steps)
    q_start = rank * shard
    cur, nxt = 0, 1
    if n_vis == 0:
        out.zero_()
        if lse is not None:
            lse.fill_(float("-inf"))
    for s in steps:
        handle = None
        if exchange is not None and s.t < world - 1:
            handle = exchange.post(list(kv_bufs[cur]), list(kv_bufs[nxt]))
        kb, vb = kv_bufs[cur]
        if s.visible:
            k_start = s.block * shard
            if n_vis == 1:
                attend(q, kb, vb, out, lse, q_start, k_start, None)
            elif s.first:
                attend(q, kb, vb, acc, lacc, q_start, k_start, None)
            elif s.last:
                attend(q, kb, vb, out, lse if lse is not None else lacc, q_start, k_start, (acc, lacc))
            else:
                attend(q, kb, vb, acc, lacc, q_start, k_start, (acc, lacc))
        if handle is not None:
            for h in handle:
                h.wait()
        cur, nxt = nxt, cur
    return out, lse


def librcx_attend(inv_freq, temperature: float, window: int, n_sink: int):
    """``attend`` for ring_forward, bound to librcx: the tensor-core (bf16,
    d = 128) or SIMT attention with the query rotation fused in its tile load;
    a previous partial is merged in the kernel's epilogue."""
    from . import _lib

    _lib.load()

    def attend(q, kb, vb, o, l, q_start, k_start, prev):
        kw = dict(window=window, n_sink=n_sink, temperature=temperature, q_start=q_start, k_start=k_start,
                  inv_freq=inv_freq, rope_flags=_lib.ROTATE_Q)
        if prev is None:
            _lib.attn_blockwise_fwd(q, kb, vb, o, l, **kw)
        else:
            _lib.attn_blockwise_merge_fwd(q, kb, vb, o, l, prev[0], prev[1], **kw)

    return attend


def rotate_key_shard(k: torch.Tensor, inv_freq, start: int, out: torch.Tensor) -> torch.Tensor:
    """Rotate a key shard whose row n is global token start + n (librcx
    rope_apply with explicit positions) into ``out``."""
    from . import _lib

    pos = torch.arange(start, start + k.shape[1], dtype=torch.int64, device=k.device)
    _lib.rope_apply(None, k, inv_freq, positions=pos, k_out=out)
    return out


def ring_buffers(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, inv_freq, start: int):
    """Device buffers of one rank: the two (k, v) block buffers, with this
    rank's rotated keys and its values in the first, and the fp32 accumulator
    with its LSE."""
    B, Ns, Hq, d = q.shape
    kv_bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
    rotate_key_shard(k, inv_freq, start, kv_bufs[0][0])
    kv_bufs[0][1].copy_(v)
    acc = torch.empty(B, Ns, Hq, d, dtype=torch.float32, device=q.device)
    lacc = torch.empty(B, Hq, Ns, dtype=torch.float32, device=q.device)
    return kv_bufs, acc, lacc


def ring_attention_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, inv_freq, temperature: float = 1.0,
                        window: int = 0, n_sink: int = 0, group=None, out: Optional[torch.Tensor] = None,
                        lse: Optional[torch.Tensor] = None):
    """Ring Attention forward of this rank's shard over all ranks of ``group``
    (torch.distributed, NCCL on GPUs), with librcx kernels for the K rotation,
    the per-block attention (Q rotated in its tile load) and the LSE merge.

    q: [B, Ns, Hq, d], k, v: [B, Ns, Hkv, d] on this rank's GPU; every rank
    passes the same shapes.  Returns (out [B, Ns, Hq, d], lse [B, Hq, Ns])."""
    import torch.distributed as dist

    if not q.is_cuda:
        raise RuntimeError("ring_attention_dist runs on CUDA tensors")
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, Ns, Hq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Ns, dtype=torch.float32, device=q.device)
    attend = librcx_attend(inv_freq, temperature, window, n_sink)
    kv_bufs, acc, lacc = ring_buffers(q, k, v, inv_freq, rank * Ns)
    exch = Exchange(group) if world > 1 else None
    return ring_forward(q, kv_bufs, rank=rank, world=world, window=window, n_sink=n_sink, attend=attend,
                        exchange=exch, out=out, lse=lse, acc=acc, lacc=lacc)

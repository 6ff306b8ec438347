"""One pass of the hot path for a named workload, through the C ABI.

run_workload(w, q, k, v) prepares the call (frequencies, output and workspace
buffers, the rotated-K buffer) and returns a closure that launches one full
pass: K rotation (memory-bound), tensor-core attention with the Q rotation
fused into its tile load, and -- for ring workloads -- the ring schedule with
its LSE merges.  Nothing is computed here; every step runs in librcx kernels.
"""

from __future__ import annotations

import torch

from . import _lib


def run_workload(w, q, k, v, o=None, lse=None):
    inv, t = _lib.rope_freqs(w.scheme, w.base, w.d, w.L_train, w.L_target, w.alpha, w.beta)
    B, N, Hq, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    flags = _lib.ROTATE_Q | _lib.ROTATE_K
    if w.ring:
        need = _lib.ring_workspace_size(q, k, w.kv_block, flags)
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)

        def run():
            return _lib.ring_attn_fwd(q, k, v, o, lse, kv_block=w.kv_block, window=w.window, n_sink=w.n_sink,
                                      temperature=t, inv_freq=inv, rope_flags=flags, workspace=ws)
        return run

    if q.dtype == torch.bfloat16:
        # the tensor-core path rotates Q in its tile load; K (shared by the
        # G query heads of a group and by every query tile) is rotated once
        k_rot = torch.empty_like(k)

        def run():
            _lib.rope_apply(None, k, inv, k_out=k_rot)
            return _lib.attn_blockwise_fwd(q, k_rot, v, o, lse, kv_block=w.kv_block, window=w.window,
                                           n_sink=w.n_sink, temperature=t, inv_freq=inv,
                                           rope_flags=_lib.ROTATE_Q)
        return run

    def run():
        return _lib.attn_blockwise_fwd(q, k, v, o, lse, kv_block=w.kv_block, window=w.window, n_sink=w.n_sink,
                                       temperature=t, inv_freq=inv, rope_flags=flags)
    return run

"""The allocation-free ring forward (rcx_ring_attn_fwd_noalloc).

Some callers cannot allocate device memory -- a framework whose caching
allocator owns the device heap, or a serving loop with a fixed budget where
cudaMalloc's device synchronisation is not allowed -- so they cannot pass a
workspace.  This entry point uses the library's static device scratch instead.
Here it is called through the C ABI and compared with the workspace entry
point, rcx_ring_attn_fwd, on two calls in a row with different inputs and
shapes (the second must not see the first call's leftovers), and a request
larger than the static scratch must be refused before any launch.

The file name sorts last so that a run stopping at the first failure has run
every other test before this one.
"""

import pytest
import torch

from rope_context_extension_scaled_b200 import _lib
from rope_context_extension_scaled_b200.inputs import make_qkv
from tests._parity import TOL_BF16_O_MAX, TOL_BF16_O_MEAN, TOL_BF16_LSE_MEAN

pytestmark = pytest.mark.gpu

FLAGS = _lib.ROTATE_Q | _lib.ROTATE_K


def _compare(N, Hq, Hkv, kv_block, window, n_sink, seed):
    q, k, v = make_qkv(1, N, Hq, Hkv, 128, torch.bfloat16, seed=seed, device="cuda")
    inv, t = _lib.rope_freqs(_lib.NTK, 5e5, 128, 1024, 8192)
    need = _lib.ring_workspace_size(q, k, kv_block, FLAGS)
    assert need <= _lib.NOALLOC_SCRATCH_BYTES
    o_ref, l_ref = _lib.ring_attn_fwd(q, k, v, kv_block=kv_block, window=window, n_sink=n_sink, temperature=t,
                                      inv_freq=inv, rope_flags=FLAGS)
    o = torch.empty_like(q)
    lse = torch.empty(1, Hq, N, dtype=torch.float32, device="cuda")
    _lib.ring_attn_fwd_noalloc(q, k, v, o, lse, kv_block=kv_block, window=window, n_sink=n_sink, temperature=t,
                               inv_freq=inv, rope_flags=FLAGS)
    torch.cuda.synchronize()
    d = (o.float() - o_ref.float()).abs()
    assert d.max().item() <= TOL_BF16_O_MAX
    assert d.mean().item() <= TOL_BF16_O_MEAN
    fin = torch.isfinite(l_ref)
    assert torch.equal(torch.isneginf(lse), torch.isneginf(l_ref))
    assert (lse[fin] - l_ref[fin]).abs().mean().item() <= TOL_BF16_LSE_MEAN


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    _compare(N=4096, Hq=8, Hkv=2, kv_block=1024, window=0, n_sink=0, seed=21)
    _compare(N=2000, Hq=4, Hkv=1, kv_block=512, window=700, n_sink=4, seed=22)


def test_noalloc_refuses_requests_beyond_the_static_scratch():
    N, Hq, Hkv = 65536, 16, 2
    q = torch.empty(1, N, Hq, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(1, N, Hkv, 128, dtype=torch.bfloat16, device="cuda")
    assert _lib.ring_workspace_size(q, k, 8192, FLAGS) > _lib.NOALLOC_SCRATCH_BYTES
    o = torch.empty_like(q)
    inv, t = _lib.rope_freqs(_lib.PLAIN, 1e4, 128, 10, 10)
    with pytest.raises(_lib.RcxError) as e:
        _lib.ring_attn_fwd_noalloc(q, k, k, o, None, kv_block=8192, inv_freq=inv, rope_flags=FLAGS)
    assert e.value.status == _lib.RCX_ERR_UNSUPPORTED

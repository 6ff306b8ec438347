"""GPU parity of each C-ABI call against the float64 oracle (small and ragged
shapes that span several tiles, plus edge cases).  Calls go through the
ctypes binding of librcx.so."""

import math

import mpmath
import numpy as np
import pytest
import torch

from oracle import rcx_oracle as orc
from rope_context_extension_scaled_b200 import _lib
from rope_context_extension_scaled_b200.inputs import make_qkv
from tests._parity import (schedule, all_rows, assert_bf16, assert_f32, errors, gather_gpu, np64, oracle_rows)

pytestmark = pytest.mark.gpu

DEV = "cuda"


# ------------------------------------------------------------------ rope_apply

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,Hq,Hkv,d", [(37, 3, 1, 64), (300, 8, 2, 128), (1, 1, 1, 128)])
@pytest.mark.parametrize("pos_kind", ["arange", "random"])
def test_rope_apply_matches_oracle(dtype, N, Hq, Hkv, d, pos_kind):
    q, k, _ = make_qkv(2, N, Hq, Hkv, d, dtype, seed=1, device=DEV)
    inv, _, oinv, _ = schedule(_lib.NTK, 5e5, d, 8192, 8192 * 128)
    pos = None
    p_np = np.arange(N)
    if pos_kind == "random":
        g = torch.Generator(device=DEV)
        g.manual_seed(3)
        pos = torch.randint(0, 1 << 20, (N,), generator=g, device=DEV, dtype=torch.int64)
        p_np = pos.cpu().numpy()
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    _lib.rope_apply(q, k, inv, positions=pos, q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    for x, y in ((q, qo), (k, ko)):
        for b in range(2):
            ref = orc.rope_rotate(np64(x[b]), p_np, oinv)
            got = np64(y[b])
            if dtype == torch.float32:
                assert np.abs(got - ref).max() < 1e-5
            else:   # one bf16 rounding of the fp32 result
                assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)


def test_rope_apply_in_place_equals_out_of_place():
    q, k, _ = make_qkv(1, 257, 4, 2, 128, torch.bfloat16, seed=2, device=DEV)
    inv, _, oinv, _ = schedule(_lib.YARN, 1e4, 128, 4096, 32768)
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    _lib.rope_apply(q, k, inv, q_out=qo, k_out=ko)
    q2, k2 = q.clone(), k.clone()
    _lib.rope_apply(q2, k2, inv)
    torch.cuda.synchronize()
    assert torch.equal(q2, qo) and torch.equal(k2, ko)
    # K only
    k3 = k.clone()
    _lib.rope_apply(None, k3, inv)
    assert torch.equal(k3, ko)


def test_rope_angle_error_at_one_million():
    # Unit vectors (1, 0) in every pair, rotated in fp32: the applied angle
    # must be within 1e-5 rad of m * theta' (exact, 60-digit arithmetic).
    d = 128
    inv, _, oinv, _ = schedule(_lib.NTK, 5e5, d, 8192, 1 << 20)
    ms = [0, 1, 65535, 999_999, 1_048_575, (1 << 24) - 1]
    x = torch.zeros(1, len(ms), 1, d, dtype=torch.float32, device=DEV)
    x[..., 0::2] = 1.0
    pos = torch.tensor(ms, dtype=torch.int64, device=DEV)
    _lib.rope_apply(x, None, inv, positions=pos)
    out = x[0, :, 0].cpu().numpy().astype(np.float64)
    got = np.arctan2(out[:, 1::2], out[:, 0::2])
    mpmath.mp.dps = 60
    worst = 0.0
    for r, m in enumerate(ms):
        for i in range(d // 2):
            e = mpmath.mpf(m) * mpmath.mpf(float(inv[i]))
            ex = float(e - 2 * mpmath.pi * mpmath.nint(e / (2 * mpmath.pi)))
            diff = abs((got[r, i] - ex + math.pi) % (2 * math.pi) - math.pi)
            worst = max(worst, diff)
    assert worst <= 1e-5, worst
    assert worst <= 2e-6, worst      # observed: fp32 sincos of the fp64-reduced angle


@pytest.mark.parametrize("d", [128, 64])
def test_rope_dense_angle_error_near_one_million(d):
    # Dense layout, positions == NULL (position = token index), fp32 unit
    # vectors (1, 0) in every pair, N = 2^20 tokens of one head: the applied
    # angle of every pair must be within 1e-5 rad of m * theta' (40-digit
    # arithmetic), for the last 192 tokens below m = 1,048,575, the first 40
    # and 96 random ones.  Each token's angles are computed on their own
    # (float64 product and reduction, fp32 sincos), so the bound that holds is
    # the one of a single sincos: 2e-6.
    N = 1 << 20
    inv, _, _, _ = schedule(_lib.NTK, 5e5, d, 8192, 1 << 20)
    x = torch.zeros(1, N, 1, d, dtype=torch.float32, device=DEV)
    x[..., 0::2] = 1.0
    _lib.rope_apply(x, None, inv)
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    toks = np.unique(np.concatenate([np.arange(N - 192, N), np.arange(0, 40),
                                     rng.integers(0, N, size=96)]))
    out = x[0, torch.as_tensor(toks, device=DEV), 0].cpu().numpy().astype(np.float64)
    got = np.arctan2(out[:, 1::2], out[:, 0::2])
    mpmath.mp.dps = 40
    two_pi = 2 * mpmath.pi
    worst = 0.0
    for r, m in enumerate(toks):
        for i in range(d // 2):
            e = mpmath.mpf(int(m)) * mpmath.mpf(float(inv[i]))
            ex = float(e - two_pi * mpmath.nint(e / two_pi))
            diff = abs((got[r, i] - ex + math.pi) % (2 * math.pi) - math.pi)
            worst = max(worst, diff)
    print(f"dense rope_apply d={d}: worst angle error {worst:.3e} rad over {len(toks)} tokens")
    assert worst <= 1e-5, worst
    assert worst <= 2e-6, worst


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 96), (torch.bfloat16, 8), (torch.float32, 256),
                                     (torch.float32, 4), (torch.bfloat16, 128)])
def test_rope_apply_strided_views_and_odd_widths(dtype, d):
    # Q and K as head slices of one packed [B, N, Hq + 2 Hkv, d] tensor (row
    # stride != H * d), outputs into [B, H, N, d] storage seen as [B, N, H, d]
    # (head stride N * d); Hq + Hkv = 11 heads, so one thread's group of heads
    # straddles the Q/K boundary; head widths whose 16-byte pieces per head
    # (12, 1, 64, 1, 16) give CTAs of 252, 256, 256, 256 and 256 threads.
    B, N, Hq, Hkv = 3, 45, 8, 3
    g = torch.Generator(device="cpu")
    g.manual_seed(41)
    qkv = torch.randn(B, N, Hq + 2 * Hkv, d, generator=g).to(dtype).to(DEV)
    q, k = qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv]
    qo = torch.empty(B, Hq, N, d, dtype=dtype, device=DEV).transpose(1, 2)
    ko = torch.empty(B, Hkv, N, d, dtype=dtype, device=DEV).transpose(1, 2)
    inv, _, oinv, _ = schedule(_lib.YARN, 1e4, d, 4096, 65536)
    pos = torch.randint(0, 1 << 17, (N,), generator=g, dtype=torch.int64).to(DEV)
    v_before = qkv[:, :, Hq + Hkv:].clone()
    _lib.rope_apply(q, k, inv, positions=pos, q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    p_np = pos.cpu().numpy()
    for x, y in ((q, qo), (k, ko)):
        for b in range(B):
            ref = orc.rope_rotate(np64(x[b]), p_np, oinv)
            got = np64(y[b])
            if dtype == torch.float32:
                assert np.abs(got - ref).max() < 1e-5
            else:
                assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)
    # the V slice of the packed tensor is not written
    assert torch.equal(qkv[:, :, Hq + Hkv:], v_before)


def test_rope_apply_rejects_misaligned():
    q = torch.zeros(1, 4, 1, 130, dtype=torch.bfloat16, device=DEV)[..., 1:129]   # 2-byte offset
    inv, _, oinv, _ = schedule(_lib.PLAIN, 1e4, 128, 10, 10)
    with pytest.raises(_lib.RcxError) as e:
        _lib.rope_apply(q, None, inv)
    assert e.value.status == _lib.RCX_ERR_ALIGNMENT


# ------------------------------------------------------------------ attention

def _run_attn(q, k, v, inv, t, rows=None, **kw):
    o, lse = _lib.attn_blockwise_fwd(q, k, v, temperature=t, inv_freq=inv, **kw)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("N,kv_block,window,n_sink", [
    (512, 64, 0, 0), (200, 0, 0, 0), (333, 50, 40, 3), (97, 7, 0, 0), (130, 0, 16, 0)])
def test_fp32_attention_fused_rope(N, kv_block, window, n_sink):
    q, k, v = make_qkv(1, N, 2, 1, 64, torch.float32, seed=4, device=DEV)
    inv, t, oinv, ot = schedule(_lib.PI, 1e4, 64, 256, 512)
    o, lse = _run_attn(q, k, v, inv, t, kv_block=kv_block, window=window, n_sink=n_sink,
                       rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
    rows = all_rows(N, 2)
    Or, Lr = oracle_rows(q[0], k[0], v[0], oinv, ot, rows, window, n_sink)
    assert_f32(errors(*gather_gpu(o, lse, rows), Or, Lr))


@pytest.mark.parametrize("N,Hq,Hkv", [(1, 2, 1), (100, 4, 2), (128, 2, 2), (300, 8, 2), (513, 3, 1),
                                      (640, 4, 4), (257, 6, 3)])
def test_bf16_tensor_core_attention(N, Hq, Hkv):
    q, k, v = make_qkv(1, N, Hq, Hkv, 128, torch.bfloat16, seed=5, device=DEV)
    inv, t, oinv, ot = schedule(_lib.NTK, 5e5, 128, 8192, 32768)
    krot = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, k_out=krot)
    o, lse = _run_attn(q, krot, v, inv, t, rope_flags=_lib.ROTATE_Q)
    rows = all_rows(N, Hq)
    Or, Lr = oracle_rows(q[0], k[0], v[0], oinv, ot, rows)
    assert_bf16(errors(*gather_gpu(o, lse, rows), Or, Lr))


@pytest.mark.parametrize("window,n_sink,kv_block", [(64, 4, 0), (200, 0, 256), (1000, 2, 0), (129, 130, 384),
                                                    (0, 0, 384), (0, 0, 100)])
def test_bf16_window_sinks_ring_order(window, n_sink, kv_block):
    N = 777
    q, k, v = make_qkv(1, N, 4, 2, 128, torch.bfloat16, seed=6, device=DEV)
    inv, t, oinv, ot = schedule(_lib.YARN, 1e4, 128, 256, 2048)
    krot = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, k_out=krot)
    o, lse = _run_attn(q, krot, v, inv, t, rope_flags=_lib.ROTATE_Q, window=window, n_sink=n_sink,
                       kv_block=kv_block)
    rows = all_rows(N, 4)
    Or, Lr = oracle_rows(q[0], k[0], v[0], oinv, ot, rows, window, n_sink)
    assert_bf16(errors(*gather_gpu(o, lse, rows), Or, Lr))


def test_bf16_offsets_positions_and_fp32_output():
    # q rows are global tokens 500.., keys 0..; custom positions; fp32 output.
    Nq, Nk = 200, 700
    q, _, _ = make_qkv(1, Nq, 4, 2, 128, torch.bfloat16, seed=7, device=DEV)
    _, k, v = make_qkv(1, Nk, 4, 2, 128, torch.bfloat16, seed=8, device=DEV)
    g = torch.Generator(device=DEV)
    g.manual_seed(9)
    pos = torch.randint(0, 1 << 20, (Nk,), generator=g, device=DEV, dtype=torch.int64)
    inv, t, oinv, ot = schedule(_lib.DYN_NTK, 5e5, 128, 8192, 131072)
    krot = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, positions=pos, k_out=krot)
    o, lse = _run_attn(q, krot, v, inv, t, rope_flags=_lib.ROTATE_Q, q_start=500, k_start=0, positions=pos,
                       out_dtype=torch.float32)
    assert o.dtype == torch.float32
    rows = all_rows(Nq, 4)
    Or, Lr = oracle_rows(q[0], k[0], v[0], oinv, ot, rows, positions=pos, q_start=500, k_start=0)
    assert_bf16(errors(*gather_gpu(o, lse, rows), Or, Lr))


def test_bf16_attention_with_per_plane_factors():
    # LongRoPE application: an arbitrary per-plane factor vector flows
    # through K rotation and the fused Q rotation like any other schedule.
    N = 600
    q, k, v = make_qkv(1, N, 4, 2, 128, torch.bfloat16, seed=17, device=DEV)
    rng = np.random.default_rng(5)
    lam = np.exp(rng.uniform(0.0, np.log(32.0), size=64))
    inv = _lib.rope_freqs_per_pair(5e5, 128, lam)
    krot = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, k_out=krot)
    o, lse = _run_attn(q, krot, v, inv, 1.0, rope_flags=_lib.ROTATE_Q)
    rows = all_rows(N, 4)
    Or, Lr = oracle_rows(q[0], k[0], v[0], orc.rope_freqs_per_pair(5e5, 128, lam), 1.0, rows)
    assert_bf16(errors(*gather_gpu(o, lse, rows), Or, Lr))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fully_masked_rows_and_empty_inputs(dtype):
    d = 128 if dtype == torch.bfloat16 else 64
    q, k, v = make_qkv(1, 64, 2, 1, d, dtype, seed=10, device=DEV)
    # keys all after the queries: nothing visible
    o, lse = _lib.attn_blockwise_fwd(q, k, v, q_start=0, k_start=1000)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    # empty query set is a no-op
    e = q[:, :0]
    o2, l2 = _lib.attn_blockwise_fwd(e, k, v)
    assert o2.shape[1] == 0


def test_rotate_k_in_kernel_unsupported_on_tensor_core_path():
    q, k, v = make_qkv(1, 16, 2, 1, 128, torch.bfloat16, seed=11, device=DEV)
    inv, t, oinv, ot = schedule(_lib.PLAIN, 1e4, 128, 10, 10)
    with pytest.raises(_lib.RcxError) as e:
        _lib.attn_blockwise_fwd(q, k, v, inv_freq=inv, rope_flags=_lib.ROTATE_K)
    assert e.value.status == _lib.RCX_ERR_UNSUPPORTED


# ---------------------------------------------------------------------- merge

@pytest.mark.parametrize("out", ["inplace", "bf16", "f32"])
def test_merge_partials(out):
    g = torch.Generator(device=DEV)
    g.manual_seed(12)
    B, N, H, d = 2, 77, 3, 128
    oa = torch.randn(B, N, H, d, generator=g, device=DEV)
    ob = torch.randn(B, N, H, d, generator=g, device=DEV)
    la = torch.randn(B, H, N, generator=g, device=DEV) * 5
    lb = torch.randn(B, H, N, generator=g, device=DEV) * 5
    la[0, 0, :5] = -math.inf
    lb[0, 0, 3:8] = -math.inf
    ro, rl = orc.merge(np64(oa).transpose(0, 2, 1, 3), np64(la), np64(ob).transpose(0, 2, 1, 3), np64(lb))
    ro = ro.transpose(0, 2, 1, 3)
    if out == "inplace":
        oa2, la2 = oa.clone(), la.clone()
        go, gl = _lib.merge_partials(oa2, la2, ob, lb)
    else:
        dt = torch.bfloat16 if out == "bf16" else torch.float32
        go = torch.empty(B, N, H, d, dtype=dt, device=DEV)
        gl = torch.empty(B, H, N, device=DEV)
        _lib.merge_partials(oa, la, ob, lb, go, gl)
    torch.cuda.synchronize()
    tol = 1e-5 if out != "bf16" else 2e-2
    assert np.abs(np64(go) - ro).max() <= tol
    fin = np.isfinite(rl)
    assert np.array_equal(np.isneginf(np64(gl)), np.isneginf(rl))
    assert np.abs(np64(gl)[fin] - rl[fin]).max() <= 1e-5


@pytest.mark.parametrize("dtype,d,out_bf16", [(torch.bfloat16, 128, True), (torch.bfloat16, 128, False),
                                              (torch.float32, 64, False)])
def test_attention_merged_into_previous_partial(dtype, d, out_bf16):
    # Three key blocks visited in ring order 2, 1, 0 for query rows of block 2:
    # the first call writes the fp32 accumulator, the second merges in place
    # in the epilogue, the third merges into the final output.
    N, nb = 600, 200
    q, k, v = make_qkv(1, N, 4, 2, d, dtype, seed=33, device=DEV)
    inv, t, oinv, ot = schedule(_lib.YARN, 1e4, d, 256, 2048)
    krot = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, k_out=krot)
    qs = q[:, 2 * nb:].contiguous()
    acc = torch.empty(1, nb, 4, d, dtype=torch.float32, device=DEV)
    lacc = torch.empty(1, 4, nb, dtype=torch.float32, device=DEV)
    out = torch.empty(1, nb, 4, d, dtype=torch.bfloat16 if out_bf16 else torch.float32, device=DEV)
    lse = torch.empty(1, 4, nb, dtype=torch.float32, device=DEV)
    kw = dict(window=300, n_sink=3, temperature=t, q_start=2 * nb, inv_freq=inv, rope_flags=_lib.ROTATE_Q)
    blk = lambda x, b: x[:, b * nb:(b + 1) * nb].contiguous()
    _lib.attn_blockwise_fwd(qs, blk(krot, 2), blk(v, 2), acc, lacc, k_start=2 * nb, **kw)
    _lib.attn_blockwise_merge_fwd(qs, blk(krot, 1), blk(v, 1), acc, lacc, acc, lacc, k_start=nb, **kw)
    _lib.attn_blockwise_merge_fwd(qs, blk(krot, 0), blk(v, 0), out, lse, acc, lacc, k_start=0, **kw)
    torch.cuda.synchronize()
    rows = all_rows(nb, 4)
    Or, Lr = oracle_rows(qs[0], k[0], v[0], oinv, ot, rows, 300, 3, q_start=2 * nb, k_start=0)
    err = errors(*gather_gpu(out, lse, rows), Or, Lr)
    (assert_bf16 if (dtype == torch.bfloat16 or out_bf16) else assert_f32)(err)


# ----------------------------------------------------------------------- ring

@pytest.mark.parametrize("dtype,d,N,kv_block,window,n_sink", [
    (torch.bfloat16, 128, 1024, 256, 0, 0), (torch.bfloat16, 128, 1000, 384, 300, 4),
    (torch.float32, 64, 512, 64, 0, 0), (torch.float32, 64, 300, 128, 50, 2)])
def test_ring_driver_matches_oracle(dtype, d, N, kv_block, window, n_sink):
    q, k, v = make_qkv(1, N, 4, 2, d, dtype, seed=13, device=DEV)
    inv, t, oinv, ot = schedule(_lib.NTK, 1e4, d, 256, 1024)
    o, lse = _lib.ring_attn_fwd(q, k, v, kv_block=kv_block, window=window, n_sink=n_sink, temperature=t,
                                inv_freq=inv, rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
    torch.cuda.synchronize()
    rows = all_rows(N, 4)
    Or, Lr = oracle_rows(q[0], k[0], v[0], oinv, ot, rows, window, n_sink)
    err = errors(*gather_gpu(o, lse, rows), Or, Lr)
    (assert_bf16 if dtype == torch.bfloat16 else assert_f32)(err)


def test_ring_equals_single_call_bf16():
    N = 1024
    q, k, v = make_qkv(1, N, 4, 2, 128, torch.bfloat16, seed=14, device=DEV)
    inv, t, oinv, ot = schedule(_lib.NTK, 5e5, 128, 256, 2048)
    o1, l1 = _lib.ring_attn_fwd(q, k, v, kv_block=256, temperature=t, inv_freq=inv,
                                rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
    krot = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, k_out=krot)
    o2, l2 = _lib.attn_blockwise_fwd(q, krot, v, temperature=t, inv_freq=inv, rope_flags=_lib.ROTATE_Q)
    torch.cuda.synchronize()
    # same arithmetic up to the merge points: differences are bf16 output roundings
    assert (o1.float() - o2.float()).abs().max().item() <= 2 ** -7
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_ring_host_buffers_entry_point():
    N = 512
    q, k, v = make_qkv(1, N, 4, 2, 128, torch.bfloat16, seed=15, device="cpu")
    inv, t, oinv, ot = schedule(_lib.NTK, 5e5, 128, 256, 1024)
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty(1, 4, N, dtype=torch.float32).pin_memory()
    _lib.ring_attn_fwd_host(qh, kh, vh, oh, lh, kv_block=128, temperature=t, inv_freq=inv,
                            rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
    od, ld = _lib.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), kv_block=128, temperature=t, inv_freq=inv,
                                rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
    torch.cuda.synchronize()
    assert torch.equal(oh, od.cpu()) and torch.equal(lh, ld.cpu())


@pytest.mark.parametrize("B,N,Hq,Hkv,d,dtype,kv,window,n_sink,use_pos", [
    (2, 700, 4, 2, 128, torch.bfloat16, 128, 100, 3, True),     # ragged last block, batch 2, mask, positions
    (1, 300, 2, 1, 64, torch.float32, 64, 0, 0, False),         # fp32 path: K rotated in the kernel
    (1, 256, 4, 1, 128, torch.bfloat16, 0, 0, 0, False),        # one block
])
def test_ring_host_pipeline_matches_device_path(B, N, Hq, Hkv, d, dtype, kv, window, n_sink, use_pos):
    # The host entry point streams shard r's Q and V rows in, and shard r's
    # output out, on copy streams joined to the schedule by events: the result
    # must be the device-buffer result, bit for bit.
    q, k, v = make_qkv(B, N, Hq, Hkv, d, dtype, seed=17, device="cpu")
    inv, t, _, _ = schedule(_lib.YARN, 1e4, d, 128, 1024)
    pos = None
    if use_pos:
        g = torch.Generator(device="cpu")
        g.manual_seed(5)
        pos = torch.randint(0, 1 << 20, (N,), generator=g, dtype=torch.int64)
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty(B, Hq, N, dtype=torch.float32).pin_memory()
    flags = _lib.ROTATE_Q | _lib.ROTATE_K
    _lib.ring_attn_fwd_host(qh, kh, vh, oh, lh, kv_block=kv, window=window, n_sink=n_sink, temperature=t,
                            positions=pos, inv_freq=inv, rope_flags=flags)
    od, ld = _lib.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), kv_block=kv, window=window, n_sink=n_sink,
                                temperature=t, positions=None if pos is None else pos.cuda(), inv_freq=inv,
                                rope_flags=flags)
    torch.cuda.synchronize()
    assert torch.equal(oh, od.cpu()) and torch.equal(lh, ld.cpu())


def test_ring_host_staging_kept_and_released():
    # The host entry point keeps its staging memory in a library pool between
    # calls; repeated calls, a release, and a call after it give one result.
    N = 384
    q, k, v = make_qkv(1, N, 4, 2, 128, torch.bfloat16, seed=18, device="cpu")
    inv, t, _, _ = schedule(_lib.NTK, 5e5, 128, 256, 1024)
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    outs = []
    for release in (False, False, True):
        oh = torch.empty_like(qh).pin_memory()
        lh = torch.empty(1, 4, N, dtype=torch.float32).pin_memory()
        _lib.ring_attn_fwd_host(qh, kh, vh, oh, lh, kv_block=128, temperature=t, inv_freq=inv,
                                rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
        outs.append((oh, lh))
        if release:
            _lib.release_staging()
    oh, lh = torch.empty_like(qh).pin_memory(), torch.empty(1, 4, N, dtype=torch.float32).pin_memory()
    _lib.ring_attn_fwd_host(qh, kh, vh, oh, lh, kv_block=128, temperature=t, inv_freq=inv,
                            rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
    outs.append((oh, lh))
    for o_, l_ in outs[1:]:
        assert torch.equal(o_, outs[0][0]) and torch.equal(l_, outs[0][1])


# ------------------------------------------------------------ bounded waits

def test_bounded_wait_timeout_reports_and_context_survives():
    q, k, v = make_qkv(1, 256, 2, 1, 128, torch.bfloat16, seed=16, device=DEV)
    assert _lib.device_status() == 0
    _lib.debug_inject_wait_timeout(20000)
    try:
        _lib.attn_blockwise_fwd(q, k, v)
        torch.cuda.synchronize()
        assert _lib.device_status() == _lib.RCX_ERR_DEVICE_TIMEOUT
    finally:
        _lib.debug_inject_wait_timeout(0)
    # the context still works and the next run is clean
    o, lse = _lib.attn_blockwise_fwd(q, k, v)
    torch.cuda.synchronize()
    assert _lib.device_status() == 0
    assert torch.isfinite(o.float()).all()


def test_host_entry_point_reports_device_timeout():
    # The synchronous host-buffer entry point reads the device status words
    # itself: a bounded wait that ran out returns RCX_ERR_DEVICE_TIMEOUT from
    # the call, and the word is cleared for the next call.
    N = 256
    q, k, v = make_qkv(1, N, 2, 1, 128, torch.bfloat16, seed=16, device="cpu")
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    inv, t, _, _ = schedule(_lib.NTK, 5e5, 128, 256, 1024)
    assert _lib.device_status() == 0
    _lib.debug_inject_wait_timeout(20000)
    try:
        with pytest.raises(_lib.RcxError) as e:
            _lib.ring_attn_fwd_host(qh, kh, vh, oh, None, kv_block=128, temperature=t, inv_freq=inv,
                                    rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
        assert e.value.status == _lib.RCX_ERR_DEVICE_TIMEOUT
    finally:
        _lib.debug_inject_wait_timeout(0)
    assert _lib.device_status() == 0
    _lib.ring_attn_fwd_host(qh, kh, vh, oh, None, kv_block=128, temperature=t, inv_freq=inv,
                            rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
    assert torch.isfinite(oh.float()).all()


# --------------------------------------------------------------------- decode

@pytest.mark.parametrize("B,Nk,Hq,Hkv,window,n_sink,qoff", [
    (1, 1, 1, 1, 0, 0, 0), (2, 1000, 8, 1, 0, 0, 0), (1, 5000, 8, 8, 0, 0, 0), (2, 3333, 16, 4, 0, 0, 0),
    (1, 20000, 64, 8, 4096, 4, 0), (1, 777, 4, 2, 100, 3, 0), (1, 4096, 8, 2, 0, 0, 50)])
def test_decode_split_kv_matches_oracle(B, Nk, Hq, Hkv, window, n_sink, qoff):
    qf, _, _ = make_qkv(B, 1, Hq, Hkv, 128, torch.bfloat16, seed=20, device=DEV)
    _, k, v = make_qkv(B, Nk, Hq, Hkv, 128, torch.bfloat16, seed=21, device=DEV)
    inv, t, oinv, ot = schedule(_lib.NTK, 5e5, 128, 8192, 131072)
    krot = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, k_out=krot)                 # the cache holds rotated keys
    q_index = Nk - 1 + qoff                                    # newest token (or later: all keys visible)
    pos = None
    if qoff:
        pos = torch.arange(q_index + 1, dtype=torch.int64, device=DEV)
    o, lse = _lib.attn_decode_fwd(qf, krot, v, window=window, n_sink=n_sink, temperature=t, q_index=q_index,
                                  positions=pos, inv_freq=inv, rope_flags=_lib.ROTATE_Q)
    torch.cuda.synchronize()
    for b in range(B):
        rows = {h: np.array([0]) for h in range(Hq)}
        Or, Lr = oracle_rows(qf[b], k[b], v[b], oinv, ot, rows, window, n_sink, q_start=q_index, k_start=0)
        Og = {h: np64(o[b, 0, h, :])[None] for h in range(Hq)}
        Lg = {h: np.array([float(lse[b, h, 0])]) for h in range(Hq)}
        err = errors(Og, Lg, Or, Lr)
        assert err["inf_ok"] and err["o_max"] <= 2e-2 and err["lse_max"] <= 1e-3, err


@pytest.mark.parametrize("Hq,Hkv,window,n_sink", [(8, 1, 0, 0), (16, 4, 300, 2)])
def test_decode_8_byte_rows_matches_oracle(Hq, Hkv, window, n_sink):
    """K and V rows 8- but not 16-byte aligned: the SIMT decode kernel."""
    Nk = 2500
    qf, _, _ = make_qkv(1, 1, Hq, Hkv, 128, torch.bfloat16, seed=25, device=DEV)
    _, k, v = make_qkv(1, Nk, Hq, Hkv, 128, torch.bfloat16, seed=26, device=DEV)
    inv, t, oinv, ot = schedule(_lib.YARN, 1e4, 128, 4096, 32768)
    krot = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, k_out=krot)
    kp = torch.zeros(1, Nk, Hkv, 132, dtype=torch.bfloat16, device=DEV)
    vp = torch.zeros_like(kp)
    kp[..., :128] = krot
    vp[..., :128] = v
    kv, vv = kp[..., :128], vp[..., :128]                       # row stride 264 bytes
    o, lse = _lib.attn_decode_fwd(qf, kv, vv, window=window, n_sink=n_sink, temperature=t, q_index=Nk - 1,
                                  inv_freq=inv, rope_flags=_lib.ROTATE_Q)
    o2, lse2 = _lib.attn_decode_fwd(qf, krot, v, window=window, n_sink=n_sink, temperature=t, q_index=Nk - 1,
                                    inv_freq=inv, rope_flags=_lib.ROTATE_Q)
    torch.cuda.synchronize()
    rows = {h: np.array([0]) for h in range(Hq)}
    Or, Lr = oracle_rows(qf[0], k[0], v[0], oinv, ot, rows, window, n_sink, q_start=Nk - 1, k_start=0)
    for oo, ll in ((o, lse), (o2, lse2)):
        Og = {h: np64(oo[0, 0, h, :])[None] for h in range(Hq)}
        Lg = {h: np.array([float(ll[0, h, 0])]) for h in range(Hq)}
        err = errors(Og, Lg, Or, Lr)
        assert err["inf_ok"] and err["o_max"] <= 2e-2 and err["lse_max"] <= 1e-3, err


def test_decode_rejects_rotate_k_and_bad_group():
    q, k, v = make_qkv(1, 1, 6, 2, 128, torch.bfloat16, seed=22, device=DEV)   # G = 3
    _, kc, vc = make_qkv(1, 64, 6, 2, 128, torch.bfloat16, seed=23, device=DEV)
    with pytest.raises(_lib.RcxError) as e:
        _lib.attn_decode_fwd(q, kc, vc)
    assert e.value.status == _lib.RCX_ERR_UNSUPPORTED
    q2, _, _ = make_qkv(1, 1, 4, 2, 128, torch.bfloat16, seed=24, device=DEV)
    inv, _, oinv, _ = schedule(_lib.PLAIN, 1e4, 128, 10, 10)
    with pytest.raises(_lib.RcxError) as e:
        _lib.attn_decode_fwd(q2, kc, vc, inv_freq=inv, rope_flags=_lib.ROTATE_K)
    assert e.value.status == _lib.RCX_ERR_UNSUPPORTED


# ------------------------------------------------------------ batch > 1, G = 8

def _oracle_batch(q, k, v, oinv, ot, window=0, n_sink=0):
    out = []
    for b in range(q.shape[0]):
        rows = all_rows(q.shape[1], q.shape[2])
        out.append((rows, *oracle_rows(q[b], k[b], v[b], oinv, ot, rows, window, n_sink)))
    return out


@pytest.mark.parametrize("Hq,Hkv,window,n_sink", [(16, 2, 0, 0), (8, 1, 300, 4), (6, 2, 0, 0)])
def test_bf16_tensor_core_batch2(Hq, Hkv, window, n_sink):
    B, N = 2, 700
    q, k, v = make_qkv(B, N, Hq, Hkv, 128, torch.bfloat16, seed=30, device=DEV)
    inv, t, oinv, ot = schedule(_lib.YARN, 1e4, 128, 512, 4096)
    krot = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, k_out=krot)
    o, lse = _lib.attn_blockwise_fwd(q, krot, v, temperature=t, inv_freq=inv, rope_flags=_lib.ROTATE_Q,
                                     window=window, n_sink=n_sink)
    torch.cuda.synchronize()
    for b, (rows, Or, Lr) in enumerate(_oracle_batch(q, k, v, oinv, ot, window, n_sink)):
        Og = {h: np64(o[b, r, h, :]) for h, r in rows.items()}
        Lg = {h: lse[b, h, r].cpu().numpy().astype(np.float64) for h, r in rows.items()}
        assert_bf16(errors(Og, Lg, Or, Lr))


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_ring_batch2(dtype, d):
    B, N = 2, 640
    q, k, v = make_qkv(B, N, 8, 2, d, dtype, seed=31, device=DEV)
    inv, t, oinv, ot = schedule(_lib.NTK, 5e5, d, 256, 2048)
    o, lse = _lib.ring_attn_fwd(q, k, v, kv_block=256, temperature=t, inv_freq=inv,
                                rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
    torch.cuda.synchronize()
    for b, (rows, Or, Lr) in enumerate(_oracle_batch(q, k, v, oinv, ot)):
        Og = {h: np64(o[b, r, h, :]) for h, r in rows.items()}
        Lg = {h: lse[b, h, r].cpu().numpy().astype(np.float64) for h, r in rows.items()}
        (assert_bf16 if dtype == torch.bfloat16 else assert_f32)(errors(Og, Lg, Or, Lr))


def test_rope_apply_batch_wrap_in_chunk():
    # N smaller than a CTA's pass of tokens: one pass covers several batch entries.
    B, N = 5, 3
    q, k, _ = make_qkv(B, N, 2, 8, 128, torch.bfloat16, seed=32, device=DEV)
    inv, _, oinv, _ = schedule(_lib.PLAIN, 1e4, 128, 10, 10)
    ko = torch.empty_like(k)
    _lib.rope_apply(None, k, inv, k_out=ko)
    torch.cuda.synchronize()
    for b in range(B):
        ref = orc.rope_rotate(np64(k[b]), np.arange(N), oinv)
        assert np.all(np.abs(np64(ko[b]) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)

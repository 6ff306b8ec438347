"""Int8 KV cache on the GPU: codes and scales bit-exact against the oracle's
fp32 rule, and decode attention over the codes against the oracle attention
over the dequantised cache ("Context window extension: 4K to 1M" 6.1)."""

import math

import numpy as np
import pytest
import torch

from oracle import rcx_oracle as orc
from rope_context_extension_scaled_b200 import _lib
from rope_context_extension_scaled_b200.inputs import make_qkv
from tests._parity import schedule, errors, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cache(B, Nk, Hkv, seed, spread=1.0, ties=True):
    """Seeded bf16 cache: N(0,1) rows times exp(N(0, spread^2)) row magnitudes,
    a zero row and (ties=True) a row of exact rounding ties."""
    g = torch.Generator(device=DEV).manual_seed(seed)
    x = torch.randn(B, Nk, Hkv, 128, generator=g, device=DEV)
    x = (x * torch.exp(spread * torch.randn(B, Nk, Hkv, 1, generator=g, device=DEV))).to(torch.bfloat16)
    if Nk > 3:
        x[0, 1, 0] = 0.0                                   # zero row: scale 0, codes 0
        if ties:
            row = torch.zeros(128, device=DEV)
            row[:6] = torch.tensor([127.0, 2.5, -2.5, 3.5, 0.5, -126.5], device=DEV)   # exact ties (127/amax = 1)
            x[0, 2, 0] = row.to(torch.bfloat16)
    return x


# Decode caches: K rows N(0,1), the workload's distribution, so that the logit
# error from the fp16 query (relative 2^-11 per element, growing with |k|) sits
# inside the attention tolerances; V rows with spread magnitudes, so that the
# per-key V scales differ and the running s_max rescale is exercised.
def _k_cache(B, Nk, Hkv, seed):
    return _cache(B, Nk, Hkv, seed, spread=0.0, ties=False)


def _v_cache(B, Nk, Hkv, seed):
    return _cache(B, Nk, Hkv, seed, spread=0.5, ties=False)


@pytest.mark.parametrize("B,Nk,Hkv", [(1, 1, 1), (2, 1000, 8), (1, 4099, 2)])
def test_quantize_codes_and_scales_bit_exact(B, Nk, Hkv):
    x = _cache(B, Nk, Hkv, seed=50 + Nk)
    codes, scale = _lib.kv_quantize_int8(x)
    torch.cuda.synchronize()
    c_ref, s_ref = orc.quantize_kv_int8(x.float().cpu().numpy())
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(scale.permute(0, 2, 1).cpu().numpy(), s_ref)   # device scales are [B, H, N]


def test_quantize_strided_view():
    base = _cache(1, 600, 4, seed=60)
    wide = torch.zeros(1, 600, 6, 128, dtype=torch.bfloat16, device=DEV)
    wide[:, :, 1:5] = base
    x = wide[:, :, 1:5]                                    # head stride 128, token stride 768
    out = torch.zeros(1, 600, 5, 128, dtype=torch.int8, device=DEV)
    codes, scale = _lib.kv_quantize_int8(x, codes=out[:, :, :4])
    torch.cuda.synchronize()
    c_ref, s_ref = orc.quantize_kv_int8(base.float().cpu().numpy())
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(scale.permute(0, 2, 1).cpu().numpy(), s_ref)   # device scales are [B, H, N]
    assert not out[:, :, 4].any()                          # nothing written outside the view


def test_quantize_8_byte_rows_and_odd_row_count():
    # bf16 rows 8- but not 16-byte aligned take the warp-per-row kernel; 903
    # rows (not a multiple of four) exercise the ragged last group of four rows
    # of the 16-byte kernel.
    base = _cache(1, 301, 3, seed=61)
    pad = torch.zeros(1, 301, 3, 132, dtype=torch.bfloat16, device=DEV)
    pad[..., 4:] = base
    x8 = pad[..., 4:]                                      # rows start 8 bytes into 264-byte rows
    for x in (x8, base):
        codes, scale = _lib.kv_quantize_int8(x)
        torch.cuda.synchronize()
        c_ref, s_ref = orc.quantize_kv_int8(base.float().cpu().numpy())
        assert np.array_equal(codes.cpu().numpy(), c_ref)
        assert np.array_equal(scale.permute(0, 2, 1).cpu().numpy(), s_ref)   # device scales are [B, H, N]


def _oracle_decode(q, k, v, inv_freq, t, q_index, window, n_sink):
    """Oracle O [Hq, d], LSE [Hq] of one query token against an int8 cache of k, v.

    k, v: bf16 cache [Nk, Hkv, 128] (as stored); the oracle quantises them with
    its own rule and attends over code * scale."""
    kc, ks = orc.quantize_kv_int8(k.float().cpu().numpy())
    vc, vs = orc.quantize_kv_int8(v.float().cpu().numpy())
    kk = orc.dequantize_kv_int8(kc, ks)
    vv = orc.dequantize_kv_int8(vc, vs)
    qs = np64(q)                                           # [1, Hq, d]
    if inv_freq is not None:
        qs = orc.rope_rotate(qs, np.array([q_index]), inv_freq)
    Nk = kk.shape[0]
    O, L = orc.attention(qs, kk, vv, 1.0 / (math.sqrt(128) * t), window=window, n_sink=n_sink,
                         q_index=np.array([q_index]), k_index=np.arange(Nk))
    return O[0], L[:, 0]


@pytest.mark.parametrize("B,Nk,Hq,Hkv,window,n_sink,qoff", [
    (1, 1, 1, 1, 0, 0, 0), (2, 1000, 8, 1, 0, 0, 0), (1, 5000, 8, 8, 0, 0, 0), (2, 3333, 16, 4, 0, 0, 0),
    (1, 20000, 64, 8, 4096, 4, 0), (1, 777, 4, 2, 100, 3, 0), (1, 4096, 8, 2, 0, 0, 50), (1, 17, 16, 2, 0, 0, 0)])
def test_decode_int8_matches_oracle(B, Nk, Hq, Hkv, window, n_sink, qoff):
    qf, _, _ = make_qkv(B, 1, Hq, Hkv, 128, torch.bfloat16, seed=70, device=DEV)
    k = _k_cache(B, Nk, Hkv, seed=71)
    v = _v_cache(B, Nk, Hkv, seed=72)
    inv, t, oinv, ot = schedule(_lib.YARN, 5e5, 128, 8192, 131072)
    kc, ks = _lib.kv_quantize_int8(k)
    vc, vs = _lib.kv_quantize_int8(v)
    q_index = Nk - 1 + qoff
    o, lse = _lib.attn_decode_int8_fwd(qf, kc, ks, vc, vs, window=window, n_sink=n_sink, temperature=t,
                                       q_index=q_index, inv_freq=inv, rope_flags=_lib.ROTATE_Q)
    torch.cuda.synchronize()
    for b in range(B):
        Or, Lr = _oracle_decode(qf[b], k[b], v[b], oinv, ot, q_index, window, n_sink)
        Og = {h: np64(o[b, 0, h, :])[None] for h in range(Hq)}
        Lg = {h: np.array([float(lse[b, h, 0])]) for h in range(Hq)}
        Ors = {h: Or[h][None] for h in range(Hq)}
        Lrs = {h: np.array([Lr[h]]) for h in range(Hq)}
        err = errors(Og, Lg, Ors, Lrs)
        assert err["inf_ok"] and err["o_max"] <= 2e-2 and err["lse_max"] <= 1e-3, err


def test_decode_int8_fp32_output_and_matches_bf16_cache_closely():
    """fp32 O; and the int8 result stays within the quantisation error of the bf16-cache result."""
    qf, _, _ = make_qkv(1, 1, 64, 8, 128, torch.bfloat16, seed=80, device=DEV)
    _, k, v = make_qkv(1, 30000, 64, 8, 128, torch.bfloat16, seed=81, device=DEV)
    kc, ks = _lib.kv_quantize_int8(k)
    vc, vs = _lib.kv_quantize_int8(v)
    o8 = torch.empty(1, 1, 64, 128, dtype=torch.float32, device=DEV)
    _lib.attn_decode_int8_fwd(qf, kc, ks, vc, vs, o=o8)
    o16, _ = _lib.attn_decode_fwd(qf, k, v)
    torch.cuda.synchronize()
    Or, Lr = _oracle_decode(qf[0], k[0], v[0], None, 1.0, 29999, 0, 0)
    assert np.abs(o8[0, 0].double().cpu().numpy() - Or).max() <= 2e-2
    assert (o8[0, 0] - o16[0, 0].float()).abs().max().item() <= 5e-2


def test_decode_int8_full_size_cache():
    """The 1M-token cache of the decode benchmark (64 / 8 heads), every head checked."""
    Nk = 1 << 20
    qf, _, _ = make_qkv(1, 1, 64, 8, 128, torch.bfloat16, seed=90, device=DEV)
    k = _k_cache(1, Nk, 8, seed=91)
    v = _v_cache(1, Nk, 8, seed=92)
    inv, t, oinv, ot = schedule(_lib.NTK, 5e5, 128, 8192, Nk)
    kc, ks = _lib.kv_quantize_int8(k)
    vc, vs = _lib.kv_quantize_int8(v)
    o, lse = _lib.attn_decode_int8_fwd(qf, kc, ks, vc, vs, temperature=t, inv_freq=inv, rope_flags=_lib.ROTATE_Q)
    torch.cuda.synchronize()
    for g in (0, 7):                                       # KV groups 0 and 7 (query heads 0-7, 56-63)
        hs = slice(8 * g, 8 * g + 8)
        Or, Lr = _oracle_decode(qf[0][:, hs], k[0][:, g:g + 1], v[0][:, g:g + 1], oinv, ot, Nk - 1, 0, 0)
        Og = {h: np64(o[0, 0, 8 * g + h, :])[None] for h in range(8)}
        Lg = {h: np.array([float(lse[0, 8 * g + h, 0])]) for h in range(8)}
        err = errors(Og, Lg, {h: Or[h][None] for h in range(8)}, {h: np.array([Lr[h]]) for h in range(8)})
        assert err["inf_ok"] and err["o_max"] <= 2e-2 and err["lse_max"] <= 1e-3, err


def test_decode_int8_rejects_misaligned_codes():
    qf, _, _ = make_qkv(1, 1, 8, 2, 128, torch.bfloat16, seed=95, device=DEV)
    k = _cache(1, 64, 2, seed=96)
    kc, ks = _lib.kv_quantize_int8(k)
    wide = torch.zeros(1, 64, 2, 136, dtype=torch.int8, device=DEV)
    wide[..., :128] = kc
    with pytest.raises(_lib.RcxError) as e:
        _lib.attn_decode_int8_fwd(qf, wide[..., :128], ks, kc, ks)      # head stride 136 bytes
    assert e.value.status == _lib.RCX_ERR_ALIGNMENT

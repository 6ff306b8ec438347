"""Helpers of the GPU parity tests: run the library, evaluate the oracle on the
same (rounded) inputs, compare.  The oracle sees exactly the values the GPU
consumed (bf16 or fp32, upcast to float64)."""

import math

import numpy as np
import torch

from oracle import rcx_oracle as orc
from rope_context_extension_scaled_b200 import _lib

# Tolerances.  The bf16 path rounds the rotated Q and K to bf16 (u = 2^-8)
# before the tensor-core product: a logit q.k / sqrt(d) with |q|, |k| ~ sqrt(d)
# then carries an error of order sqrt(2d) u / sqrt(3) / sqrt(d) ~ 3e-3, which a
# row with very few visible keys (row 0: LSE = z_00) shows undamped.  Rows with
# many keys average it down, so the LSE gate is on the mean and the max is
# reported.
TOL_F32_MAX = 1e-4
TOL_BF16_O_MAX = 2e-2
TOL_BF16_O_MEAN = 2e-3
TOL_BF16_LSE_MEAN = 1e-3


def schedule(scheme, base, d, L_train, L_target, alpha=1.0, beta=32.0):
    """One RoPE schedule evaluated by both sides: (inv, t) from the library,
    handed to the GPU call, and (oinv, ot) from the oracle, used for the
    expected values, so an end-to-end comparison also checks the library's
    frequencies and temperature."""
    inv, t = _lib.rope_freqs(scheme, base, d, L_train, L_target, alpha, beta)
    oinv, ot = orc.rope_freqs(scheme, base, d, L_train, L_target, alpha, beta)
    return inv, t, oinv, ot


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_rows(q, k, v, inv_freq, t, rows, window=0, n_sink=0, positions=None, q_start=0, k_start=0):
    """Oracle O / LSE for the (head -> local q rows) sample, batch 0.

    q: [Nq, Hq, d], k, v: [Nk, Hkv, d] torch (any device), raw (unrotated) values.
    Only the sampled query tokens are rotated."""
    Nq, Hq, d = q.shape
    Nk = k.shape[0]
    toks = np.unique(np.concatenate([np.asarray(r) for r in rows.values()]))
    qi = q_start + toks
    kj = k_start + np.arange(Nk)
    pos = positions.cpu().numpy() if positions is not None else None
    qpos = pos[qi] if pos is not None else qi
    kpos = pos[kj] if pos is not None else kj
    qs = np64(q[torch.as_tensor(toks, device=q.device)])
    kk = np64(k)
    if inv_freq is not None:
        qs = orc.rope_rotate(qs, qpos, inv_freq)
        kk = orc.rope_rotate(kk, kpos, inv_freq)
    where = {int(tk): i for i, tk in enumerate(toks)}
    sub_rows = {h: np.array([where[int(x)] for x in r]) for h, r in rows.items()}
    O, L = orc.attention(qs, kk, np64(v), 1.0 / (math.sqrt(d) * t), window=window, n_sink=n_sink,
                         q_index=qi, k_index=kj, rows=sub_rows)
    return O, L


def gather_gpu(o, lse, rows):
    """GPU O [1, N, H, d] / LSE [1, H, N] at the sampled rows -> dicts."""
    Og, Lg = {}, {}
    for h, r in rows.items():
        idx = torch.as_tensor(r, device=o.device)
        Og[h] = np64(o[0, idx, h, :])
        Lg[h] = lse[0, h, idx].cpu().numpy().astype(np.float64)
    return Og, Lg


def errors(Og, Lg, Or, Lr):
    do = np.concatenate([np.abs(Og[h] - Or[h]).ravel() for h in Or])
    fin = [np.isfinite(Lr[h]) for h in Or]
    dl = np.concatenate([np.abs(Lg[h][f] - Lr[h][f]) for h, f in zip(Or, fin)])
    inf_ok = all(np.array_equal(np.isneginf(Lg[h]), np.isneginf(Lr[h])) for h in Or)
    return dict(o_max=float(do.max()) if do.size else 0.0, o_mean=float(do.mean()) if do.size else 0.0,
                lse_max=float(dl.max()) if dl.size else 0.0, lse_mean=float(dl.mean()) if dl.size else 0.0,
                inf_ok=inf_ok)


def all_rows(N, H):
    return {h: np.arange(N) for h in range(H)}


def assert_bf16(err):
    assert err["inf_ok"], err
    assert err["o_max"] <= TOL_BF16_O_MAX, err
    assert err["o_mean"] <= TOL_BF16_O_MEAN, err
    assert err["lse_mean"] <= TOL_BF16_LSE_MEAN, err


def assert_f32(err):
    assert err["inf_ok"], err
    assert err["o_max"] <= TOL_F32_MAX, err
    assert err["lse_max"] <= TOL_F32_MAX, err

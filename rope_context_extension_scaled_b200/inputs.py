"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

Holds none of the method's arithmetic: it only draws Q, K, V from N(0, 1) with
a seeded torch generator and rounds them to the storage dtype, and picks the
sampled query rows that the parity checks evaluate.

Recipe (all configurations): one generator seeded with ``seed`` on the target
device; Q, then K, then V, each drawn in fp32 with shape [B, N, H, d] and
rounded to the storage dtype (round to nearest even for bf16).  Positions are
0..N-1 unless a test says otherwise.
"""

from __future__ import annotations

import numpy as np
import torch


def make_qkv(B, N, Hq, Hkv, d, dtype=torch.bfloat16, seed=0, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = torch.randn(B, N, Hq, d, generator=g, device=device, dtype=torch.float32).to(dtype)
    k = torch.randn(B, N, Hkv, d, generator=g, device=device, dtype=torch.float32).to(dtype)
    v = torch.randn(B, N, Hkv, d, generator=g, device=device, dtype=torch.float32).to(dtype)
    return q, k, v


def sample_rows(N, Hq, n_rows, seed=0, must_tokens=()):
    """Seeded (head -> token array) sample of query rows for sampled parity.

    Uniform over tokens, at least n_rows // Hq per head, and every token in
    ``must_tokens`` (clipped to [0, N)) on every head.
    """
    rng = np.random.default_rng(seed)
    per_head = max(1, n_rows // Hq)
    must = np.array(sorted({int(t) for t in must_tokens if 0 <= int(t) < N}), dtype=np.int64)
    rows = {}
    for h in range(Hq):
        r = rng.integers(0, N, size=per_head)
        rows[h] = np.unique(np.concatenate([r, must]))
    return rows

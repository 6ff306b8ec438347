"""Full-size parity of the five workloads, in the launch configuration bench.py
times: every row against the oracle for the small ones, >= 4096 seeded sampled
(head, token) rows for 32K, 128K and 1M (tokens 0, 1, N-1, the ring-block and
window boundaries always included)."""

import math

import numpy as np
import pytest
import torch

from rope_context_extension_scaled_b200 import _lib
from rope_context_extension_scaled_b200.configs import ORDER, WORKLOADS
from rope_context_extension_scaled_b200.inputs import make_qkv, sample_rows
from rope_context_extension_scaled_b200.runner import run_workload
from tests._parity import schedule, all_rows, assert_bf16, assert_f32, errors, gather_gpu, oracle_rows

pytestmark = pytest.mark.gpu


def _must_tokens(w):
    must = [0, 1, w.N - 1]
    if w.kv_block:
        for j in range(w.kv_block, w.N, w.kv_block):
            must += [j - 1, j]
    if w.window:
        must += [w.window - 1, w.window, w.window + w.n_sink]
    return must


@pytest.mark.parametrize("name", ORDER)
def test_workload_parity(name):
    w = WORKLOADS[name]
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    q, k, v = make_qkv(w.B, w.N, w.Hq, w.Hkv, w.d, dt, seed=0, device="cuda")
    run = run_workload(w, q, k, v)
    o, lse = run()
    torch.cuda.synchronize()
    inv, t, oinv, ot = schedule(w.scheme, w.base, w.d, w.L_train, w.L_target, w.alpha, w.beta)
    rows = all_rows(w.N, w.Hq) if not w.sample_rows else sample_rows(w.N, w.Hq, w.sample_rows, seed=0,
                                                                       must_tokens=_must_tokens(w))
    assert sum(len(r) for r in rows.values()) >= min(4096, w.N * w.Hq)
    Or, Lr = oracle_rows(q[0], k[0], v[0], oinv, ot, rows, w.window, w.n_sink)
    err = errors(*gather_gpu(o, lse, rows), Or, Lr)
    print(name, err)
    (assert_f32 if w.dtype == "f32" else assert_bf16)(err)

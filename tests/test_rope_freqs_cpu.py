"""Host frequency schedules of the library (rcx_rope_freqs) against the oracle.

Bar: relative error <= 1e-6 on every frequency (the schedules are float64 on
both sides, so the observed error is at rounding level)."""

import numpy as np
import pytest

from oracle import rcx_oracle as orc
from rope_context_extension_scaled_b200 import _lib

CASES = [
    # scheme, base, d, L_train, L_target, alpha, beta   (the five workloads' schedules + edges)
    (orc.PI, 1e4, 64, 256, 512, 1.0, 32.0),
    (orc.NTK, 5e5, 128, 8192, 32768, 1.0, 32.0),
    (orc.YARN, 1e4, 128, 4096, 32768, 1.0, 32.0),
    (orc.NTK_PARTS, 1e4, 128, 4096, 32768, 1.0, 32.0),
    (orc.DYN_NTK, 5e5, 128, 8192, 131072, 1.0, 32.0),
    (orc.NTK, 5e5, 128, 8192, 1 << 20, 1.0, 32.0),
    (orc.PLAIN, 1e4, 128, 4096, 4096, 1.0, 32.0),
    (orc.DYN_NTK, 1e4, 64, 4096, 2048, 1.0, 32.0),     # l < L_train: plain
    (orc.NTK_PARTS, 1e4, 16, 100, 1600, 2.0, 16.0),
    (orc.YARN, 5e5, 256, 8192, 8192 * 64, 1.0, 32.0),
    (orc.PI, 1e4, 2, 10, 30, 1.0, 32.0),
]


@pytest.mark.parametrize("case", CASES)
def test_rope_freqs_match_oracle(case):
    scheme, base, d, Lt, Lg, al, be = case
    got, t = _lib.rope_freqs(scheme, base, d, Lt, Lg, al, be)
    ref, tr = orc.rope_freqs(scheme, base, d, Lt, Lg, al, be)
    np.testing.assert_allclose(got, ref, rtol=1e-6, atol=0)
    assert np.max(np.abs(got / ref - 1)) < 1e-13       # observed: rounding level
    assert abs(t - tr) < 1e-12


@pytest.mark.parametrize("bad", [
    dict(scheme=9), dict(d=3), dict(d=0), dict(base=1.0), dict(L_train=0), dict(L_target=0),
    dict(scheme=orc.NTK_PARTS, alpha=32.0, beta=1.0), dict(scheme=orc.NTK, d=2),
])
def test_rope_freqs_rejects_bad_arguments(bad):
    args = dict(scheme=orc.PLAIN, base=1e4, d=64, L_train=10, L_target=20, alpha=1.0, beta=32.0)
    args.update(bad)
    with pytest.raises(_lib.RcxError) as e:
        _lib.rope_freqs(args["scheme"], args["base"], args["d"], args["L_train"], args["L_target"],
                        args["alpha"], args["beta"])
    assert e.value.status == _lib.RCX_ERR_INVALID_ARG


@pytest.mark.parametrize("d", [2, 64, 128, 256])
def test_per_pair_factors_match_oracle(d):
    rng = np.random.default_rng(d)
    lam = np.exp(rng.uniform(0.0, np.log(64.0), size=d // 2))
    got = _lib.rope_freqs_per_pair(5e5, d, lam)
    ref = orc.rope_freqs_per_pair(5e5, d, lam)
    assert np.max(np.abs(got / ref - 1)) < 1e-13


@pytest.mark.parametrize("bad", [0.0, -1.0, float("inf"), float("nan")])
def test_per_pair_factors_reject_bad_values(bad):
    lam = np.ones(64)
    lam[7] = bad
    with pytest.raises(_lib.RcxError) as e:
        _lib.rope_freqs_per_pair(1e4, 128, lam)
    assert e.value.status == _lib.RCX_ERR_INVALID_ARG

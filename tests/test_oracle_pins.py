"""Pins of the float64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages state (tests/golden/pages_examples.json), hand derivations
(tests/golden/derived_values.json), closed forms, textbook special cases,
library routines (torch SDPA, logsumexp, mpmath) and brute force on tiny
inputs.  CPU only.
"""

import json
import math
import os

import mpmath
import numpy as np
import pytest
import torch

from oracle import rcx_oracle as orc

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


PAGES = _gold("pages_examples.json")
DERIVED = _gold("derived_values.json")


# ---------------------------------------------------------------- frequencies

def test_theta_textbook_values():
    # base^(-2i/d) with base 10000: d = 8 gives exact decades, d = 4 gives 1, 0.01.
    base = PAGES["rope_default_base"]["base"]
    np.testing.assert_allclose(orc.rope_theta(base, 8), [1.0, 0.1, 0.01, 0.001], rtol=1e-15)
    np.testing.assert_allclose(orc.rope_theta(base, 4), [1.0, 0.01], rtol=1e-15)
    np.testing.assert_array_equal(orc.rope_theta(base, 2), [1.0])
    assert orc.rope_theta(base, 128).shape == (64,)


@pytest.mark.parametrize("base,d,s", [(1e4, 128, 4.0), (5e5, 128, 4.0), (5e5, 128, 128.0),
                                      (1e4, 64, 2.0), (1e4, 16, 32.0)])
def test_ntk_exponent_fixes_highest_pair(base, d, s):
    # The d/(d-2) exponent is chosen so the lowest-frequency pair is divided by
    # exactly s while the highest-frequency pair (theta_0 = 1) is unchanged.
    th = orc.rope_theta(base, d)
    L = 1024
    ntk, t = orc.rope_freqs(orc.NTK, base, d, L, int(L * s))
    assert t == 1.0
    assert ntk[0] == 1.0
    assert abs(ntk[-1] * s / th[-1] - 1.0) < 1e-13
    # every middle pair is scaled by something strictly between 1 and 1/s
    ratio = ntk[1:-1] / th[1:-1]
    assert np.all(ratio < 1.0) and np.all(ratio > 1.0 / s)
    assert np.all(np.diff(ratio) < 0)


def test_pi_example_from_page():
    ex = PAGES["pi_4k_to_8k"]
    th = orc.rope_theta(1e4, 128)
    pi, t = orc.rope_freqs(orc.PI, 1e4, 128, ex["L_train"], ex["L_target"])
    np.testing.assert_array_equal(pi, th * ex["position_factor"])
    assert t == 1.0
    ex2 = PAGES["pi_4k_to_128k"]
    pi2, _ = orc.rope_freqs(orc.PI, 1e4, 128, ex2["L_train"], ex2["L_target"])
    np.testing.assert_allclose(th / pi2, ex2["s"], rtol=1e-15)


def test_pi_position_form_equals_frequency_form():
    # The page writes PI as m -> m/s (and m' = m L_train/L_target); the oracle
    # returns theta/s.  Both angles agree to one rounding.
    rng = np.random.default_rng(1)
    th = orc.rope_theta(1e4, 64)
    s = 2.0
    pi, _ = orc.rope_freqs(orc.PI, 1e4, 64, 256, 512)
    m = rng.integers(0, 2 ** 20, size=200).astype(np.float64)
    a1 = (m[:, None] / s) * th[None, :]
    a2 = m[:, None] * pi[None, :]
    np.testing.assert_allclose(a1, a2, rtol=4.5e-16, atol=0)


def test_dynamic_ntk_matches_static_and_plain():
    th = orc.rope_theta(5e5, 128)
    for l in (1, 4096, 8192):
        f, t = orc.rope_freqs(orc.DYN_NTK, 5e5, 128, 8192, l)
        np.testing.assert_array_equal(f, th)          # l <= L_train: factor 1.0
        assert t == 1.0
    for s in (2, 16, 128):
        dyn, _ = orc.rope_freqs(orc.DYN_NTK, 5e5, 128, 8192, 8192 * s)
        ntk, _ = orc.rope_freqs(orc.NTK, 5e5, 128, 8192, 8192 * s)
        np.testing.assert_array_equal(dyn, ntk)
    # base' at l = 131072 is base * 16^(128/126): lowest-frequency pair / 16
    dyn, _ = orc.rope_freqs(orc.DYN_NTK, 5e5, 128, 8192, 131072)
    assert abs(dyn[-1] * 16 / th[-1] - 1) < 1e-13


def test_ntk_parts_bands_hand_derived():
    ex = DERIVED["ntk_parts_bands_llama70b"]
    th = orc.rope_theta(1e4, 128)
    f, t = orc.rope_freqs(orc.NTK_PARTS, 1e4, 128, 4096, 4096 * 8, alpha=1.0, beta=32.0)
    assert t == 1.0
    a, b = ex["unscaled_pairs"]
    np.testing.assert_array_equal(f[a:b + 1], th[a:b + 1])
    a, b = ex["interpolated_pairs"]
    np.testing.assert_array_equal(f[a:b + 1], th[a:b + 1] / 8.0)
    a, b = ex["ramp_pairs"]
    ratio = f[a:b + 1] / th[a:b + 1]
    assert np.all(ratio < 1.0) and np.all(ratio > 1.0 / 8.0)
    full = f / th
    assert np.all(np.diff(full) <= 0)                 # monotone in wavelength


def test_ntk_parts_factor_continuous_at_edges():
    L, s, al, be = 4096.0, 8.0, 1.0, 32.0
    lo, hi = L / be, L / al
    eps = 1e-9
    f = lambda lam: orc.ntk_parts_factor(lam, L, s, al, be)
    assert f(lo - eps) == 1.0
    assert abs(f(lo + eps) - 1.0) < 1e-10
    assert f(hi + eps) == 1.0 / s
    assert abs(f(hi - eps) - 1.0 / s) < 1e-10
    # linear in the wavelength: the midpoint sits halfway between 1 and 1/s
    assert abs(f(0.5 * (lo + hi)) - 0.5 * (1.0 + 1.0 / s)) < 1e-15


@pytest.mark.parametrize("scheme", [orc.PLAIN, orc.PI, orc.NTK, orc.DYN_NTK, orc.NTK_PARTS, orc.YARN])
def test_s_equal_one_is_plain(scheme):
    th = orc.rope_theta(1e4, 128)
    f, t = orc.rope_freqs(scheme, 1e4, 128, 4096, 4096)
    np.testing.assert_array_equal(f, th)
    assert t == 1.0


def test_yarn_temperature_closed_forms():
    assert orc.yarn_temperature(1.0) == 1.0
    assert abs(orc.yarn_temperature(math.e) - 1.1) < 1e-15
    assert abs(orc.yarn_temperature(math.exp(10.0)) - 2.0) < 1e-15
    f, t = orc.rope_freqs(orc.YARN, 1e4, 128, 4096, 32768)
    assert abs(t - DERIVED["yarn_t"]["s8"]) < 1e-15
    f2, _ = orc.rope_freqs(orc.NTK_PARTS, 1e4, 128, 4096, 32768)
    np.testing.assert_array_equal(f, f2)


def test_per_pair_factors_reduce_to_plain_pi_and_ntk_parts():
    th = orc.rope_theta(1e4, 128)
    np.testing.assert_array_equal(orc.rope_freqs_per_pair(1e4, 128, np.ones(64)), th)
    pi, _ = orc.rope_freqs(orc.PI, 1e4, 128, 4096, 4096 * 8)
    np.testing.assert_allclose(orc.rope_freqs_per_pair(1e4, 128, np.full(64, 8.0)), pi, rtol=1e-15)
    # NTK-by-parts is a particular factor vector: lambda_i = 1 / f(lambda_i)
    parts, _ = orc.rope_freqs(orc.NTK_PARTS, 1e4, 128, 4096, 32768)
    lam = th / parts
    np.testing.assert_allclose(orc.rope_freqs_per_pair(1e4, 128, lam), parts, rtol=1e-15)
    assert lam[0] == 1.0 and lam[-1] == 8.0
    with pytest.raises(ValueError):
        orc.rope_freqs_per_pair(1e4, 128, np.zeros(64))
    with pytest.raises(ValueError):
        orc.rope_freqs_per_pair(1e4, 128, np.ones(63))


# ------------------------------------------------------------------- rotation

def test_rotation_quarter_turn_direction():
    # R(pi/2) of the textbook rotation matrix maps (1, 0) to (0, 1).
    x = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])          # two tokens, 1 head, d=2
    out = orc.rope_rotate(x, [1, 1], np.array([math.pi / 2]))
    np.testing.assert_allclose(out[0, 0], [0.0, 1.0], atol=1e-15)
    np.testing.assert_allclose(out[1, 0], [-1.0, 0.0], atol=1e-15)


def test_rotation_pairs_are_adjacent_dimensions():
    # Pair (2i, 2i+1) rotates together: with theta = (pi/2, 0) at m = 1 only
    # dimensions 0 and 1 move, and they move as a quarter turn.
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    out = orc.rope_rotate(x, [1], np.array([math.pi / 2, 0.0]))
    np.testing.assert_allclose(out[0, 0], [-2.0, 1.0, 3.0, 4.0], atol=1e-15)


def test_rotation_preserves_pair_norms():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((50, 3, 64))
    pos = rng.integers(0, 2 ** 20, size=50)
    out = orc.rope_rotate(x, pos, orc.rope_theta(1e4, 64))
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = out[..., 0::2] ** 2 + out[..., 1::2] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-13)


@pytest.mark.parametrize("delta", [1, 1000, 2 ** 16, 2 ** 20 - 100])
def test_relative_position_property(delta):
    # q_m . k_n depends only on m - n ("Context Extension", Technical principles).
    rng = np.random.default_rng(3)
    d = 128
    f, _ = orc.rope_freqs(orc.NTK, 5e5, d, 8192, 8192 * 128)
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((1, 1, d))
    for m, n in [(5, 2), (77, 77), (3, 90)]:
        a = np.dot(orc.rope_rotate(q, [m], f)[0, 0], orc.rope_rotate(k, [n], f)[0, 0])
        b = np.dot(orc.rope_rotate(q, [m + delta], f)[0, 0], orc.rope_rotate(k, [n + delta], f)[0, 0])
        # fp64 angles near 2^20 rad carry ~1e-10 absolute error per term
        assert abs(a - b) <= 1e-8 * (1 + abs(a))


def test_rotation_angle_exact_at_largest_position():
    # The angle applied at m = 1,048,575 matches m*theta mod 2pi computed in
    # 60-digit arithmetic (mpmath) to 1e-9 rad -- far inside the 1e-5 bar.
    m = 1_048_575
    f, _ = orc.rope_freqs(orc.NTK, 5e5, 128, 8192, 8192 * 128)
    x = np.zeros((1, 1, 128))
    x[0, 0, 0::2] = 1.0
    out = orc.rope_rotate(x, [m], f)[0, 0]
    got = np.arctan2(out[1::2], out[0::2])
    mpmath.mp.dps = 60
    for i in range(64):
        exact = mpmath.mpf(m) * mpmath.mpf(float(f[i]))
        r = float(exact - 2 * mpmath.pi * mpmath.nint(exact / (2 * mpmath.pi)))
        diff = (got[i] - r + math.pi) % (2 * math.pi) - math.pi
        assert abs(diff) < 1e-9, (i, diff)


# ---------------------------------------------------------------------- masks

def test_mask_truth_table_window_and_sinks():
    # w = 3 keys (i-3 < j <= i) plus sinks {0, 1}, written out by hand.
    expected = {
        0: [0], 1: [0, 1], 2: [0, 1, 2], 3: [0, 1, 2, 3], 4: [0, 1, 2, 3, 4],
        5: [0, 1, 3, 4, 5], 6: [0, 1, 4, 5, 6], 7: [0, 1, 5, 6, 7],
    }
    for i, js in expected.items():
        got = [j for j in range(8) if orc.visible(i, j, 3, 2)]
        assert got == js, (i, got)
    # no window: plain causal; sinks are ignored
    for i in range(8):
        assert [j for j in range(8) if orc.visible(i, j, 0, 2)] == list(range(i + 1))


def test_page_sink_tokens_are_first_four():
    sinks = PAGES["streaming_sinks"]["sink_tokens"]
    w = PAGES["typical_window"]["w"]
    i = 20000
    vis = [j for j in range(i + 1) if orc.visible(i, j, w, len(sinks))]
    assert vis[:4] == sinks and vis[4] == i - w + 1 and vis[-1] == i
    assert len(vis) == w + 4


def test_visible_pair_counts():
    assert orc.causal_visible_pairs(131072, 4096, 4) == DERIVED["visible_pairs_128k_window"]["pairs"]
    assert orc.causal_visible_pairs(1048576) == DERIVED["visible_pairs_1m_causal"]["pairs"]
    for N in (1, 2, 7, 64):
        assert orc.causal_visible_pairs(N) == N * (N + 1) // 2
    # brute force on small sizes
    for N, w, ns in [(13, 4, 2), (9, 1, 0), (20, 30, 3), (17, 5, 5)]:
        brute = sum(bool(orc.visible(i, j, w, ns)) for i in range(N) for j in range(N))
        assert orc.causal_visible_pairs(N, w, ns) == brute


@pytest.mark.parametrize("key", ["compute_ratio_32k_vs_4k", "compute_ratio_128k_vs_8k"])
def test_quadratic_compute_ratio_from_pages(key):
    ex = PAGES[key]
    r = orc.causal_visible_pairs(ex["n_long"]) / orc.causal_visible_pairs(ex["n_short"])
    assert abs(r / ex["ratio"] - 1) < 2e-3


# ------------------------------------------------------------------ attention

def _rand_qkv(rng, Nq, Nk, Hq, Hkv, d):
    return (rng.standard_normal((Nq, Hq, d)), rng.standard_normal((Nk, Hkv, d)),
            rng.standard_normal((Nk, Hkv, d)))


@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (4, 2), (8, 2)])
def test_attention_matches_torch_sdpa_causal(Hq, Hkv):
    rng = np.random.default_rng(4)
    N, d = 37, 16
    q, k, v = _rand_qkv(rng, N, N, Hq, Hkv, d)
    scale = 1.0 / (math.sqrt(d) * 1.2)
    O, L = orc.attention(q, k, v, scale)
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]
    tk = torch.from_numpy(k).permute(1, 0, 2)[None]
    tv = torch.from_numpy(v).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, is_causal=True, scale=scale, enable_gqa=True)[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-12)
    G = Hq // Hkv
    for h in range(Hq):
        z = (q[:, h] @ k[:, h // G].T) * scale
        z = z + np.triu(np.full((N, N), -np.inf), 1)
        np.testing.assert_allclose(L[h], torch.logsumexp(torch.from_numpy(z), dim=1).numpy(), rtol=1e-13)


def test_attention_matches_sdpa_with_handwritten_window_mask():
    rng = np.random.default_rng(5)
    N, d, w, ns = 29, 8, 5, 3
    q, k, v = _rand_qkv(rng, N, N, 2, 1, d)
    mask = np.zeros((N, N), dtype=bool)
    for i in range(N):
        for j in range(N):
            if j <= i and (i - j < w or j < ns):      # window of w keys, sinks
                mask[i, j] = True
    O, L = orc.attention(q, k, v, 0.3, window=w, n_sink=ns)
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]
    tk = torch.from_numpy(k).permute(1, 0, 2)[None]
    tv = torch.from_numpy(v).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=torch.from_numpy(mask), scale=0.3, enable_gqa=True)[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-12)


def test_zero_query_gives_mean_of_visible_values():
    # q = 0: every visible logit is 0, so O is the mean of the visible v and
    # lse = ln(#visible) -- pins the per-row mask count.
    rng = np.random.default_rng(6)
    N, d, w, ns = 40, 8, 6, 2
    q = np.zeros((N, 1, d))
    k = rng.standard_normal((N, 1, d))
    v = rng.standard_normal((N, 1, d))
    O, L = orc.attention(q, k, v, 1.0, window=w, n_sink=ns)
    for i in range(N):
        js = [j for j in range(N) if j <= i and (j > i - w or j < ns)]
        np.testing.assert_allclose(O[i, 0], v[js, 0].mean(axis=0), rtol=1e-13, atol=1e-14)
        assert abs(L[0, i] - math.log(len(js))) < 1e-14


def test_first_row_and_two_key_row():
    rng = np.random.default_rng(7)
    q, k, v = _rand_qkv(rng, 5, 5, 1, 1, 4)
    sc = 0.7
    O, L = orc.attention(q, k, v, sc)
    np.testing.assert_allclose(O[0, 0], v[0, 0], rtol=1e-15)
    assert abs(L[0, 0] - sc * q[0, 0] @ k[0, 0]) < 1e-15
    z0, z1 = sc * q[1, 0] @ k[0, 0], sc * q[1, 0] @ k[1, 0]
    p1 = 1.0 / (1.0 + math.exp(z0 - z1))                 # logistic of the gap
    np.testing.assert_allclose(O[1, 0], (1 - p1) * v[0, 0] + p1 * v[1, 0], rtol=1e-13)
    assert abs(L[0, 1] - (max(z0, z1) + math.log1p(math.exp(-abs(z0 - z1))))) < 1e-14


def test_window_not_smaller_than_sequence_is_causal():
    rng = np.random.default_rng(8)
    q, k, v = _rand_qkv(rng, 20, 20, 2, 2, 8)
    a = orc.attention(q, k, v, 0.5)
    b = orc.attention(q, k, v, 0.5, window=20, n_sink=3)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_gqa_uses_consecutive_groups():
    rng = np.random.default_rng(9)
    q, k, v = _rand_qkv(rng, 12, 12, 4, 2, 8)
    O, L = orc.attention(q, k, v, 0.4)
    for h in range(4):
        g = h // 2
        o1, l1 = orc.attention(q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1], 0.4)
        np.testing.assert_allclose(O[:, h], o1[:, 0], rtol=1e-15)


def test_sampled_rows_equal_full():
    rng = np.random.default_rng(10)
    q, k, v = _rand_qkv(rng, 30, 30, 4, 1, 8)
    O, L = orc.attention(q, k, v, 0.4, window=7, n_sink=2)
    rows = {0: np.array([0, 5, 29]), 3: np.array([12])}
    o2, l2 = orc.attention(q, k, v, 0.4, window=7, n_sink=2, rows=rows)
    for h, r in rows.items():
        # BLAS may sum in another order for a sub-matrix: equal to rounding
        np.testing.assert_allclose(o2[h], O[r, h], rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(l2[h], L[h, r], rtol=1e-14)


def test_fully_masked_row_offsets():
    # Keys after every query (k_index > q_index): nothing is visible.
    rng = np.random.default_rng(11)
    q, k, v = _rand_qkv(rng, 4, 4, 1, 1, 4)
    O, L = orc.attention(q, k, v, 1.0, q_index=np.arange(4), k_index=np.arange(10, 14))
    assert np.all(O == 0) and np.all(np.isneginf(L))


@pytest.mark.parametrize("kv_block", [1, 3, 7, 8, 16, 64])
@pytest.mark.parametrize("window,n_sink", [(0, 0), (9, 2)])
def test_blockwise_online_softmax_equals_full(kv_block, window, n_sink):
    rng = np.random.default_rng(12)
    N = 48
    q, k, v = _rand_qkv(rng, N, N, 4, 2, 8)
    full = orc.attention(q, k, v, 0.35, window=window, n_sink=n_sink)
    blocks = [np.arange(s, min(s + kv_block, N)) for s in range(0, N, kv_block)]
    got = orc.attention_blockwise(q, k, v, 0.35, window, n_sink, blocks)
    np.testing.assert_allclose(got[0], full[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(got[1], full[1], rtol=1e-12, atol=1e-13)
    # reversed (ring-like) order gives the same result
    got = orc.attention_blockwise(q, k, v, 0.35, window, n_sink, blocks[::-1])
    np.testing.assert_allclose(got[0], full[0], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------- merge

def test_merge_identities():
    rng = np.random.default_rng(13)
    o = rng.standard_normal((6, 8))
    lse = rng.standard_normal(6) * 3
    mo, ml = orc.merge(o, lse, o, lse)
    np.testing.assert_allclose(mo, o, rtol=1e-15)
    np.testing.assert_allclose(ml, lse + math.log(2.0), rtol=1e-15)
    ninf = np.full(6, -np.inf)
    mo, ml = orc.merge(o, lse, np.zeros_like(o), ninf)
    np.testing.assert_array_equal(mo, o)
    np.testing.assert_array_equal(ml, lse)
    mo, ml = orc.merge(np.zeros_like(o), ninf, np.zeros_like(o), ninf)
    assert np.all(mo == 0) and np.all(np.isneginf(ml))


def test_merge_of_disjoint_key_sets_equals_joint_softmax():
    rng = np.random.default_rng(14)
    N = 33
    q, k, v = _rand_qkv(rng, N, N, 2, 1, 8)
    full = orc.attention(q, k, v, 0.5)
    split = 13
    a = orc.attention(q, k[:split], v[:split], 0.5, k_index=np.arange(split))
    b = orc.attention(q, k[split:], v[split:], 0.5, k_index=np.arange(split, N))
    o, l = orc.merge(a[0], a[1].T, b[0], b[1].T)
    np.testing.assert_allclose(o, full[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l.T, full[1], rtol=1e-13)
    # commutative, associative
    o2, l2 = orc.merge(b[0], b[1].T, a[0], a[1].T)
    np.testing.assert_allclose(o2, o, rtol=1e-14, atol=1e-15)
    c = orc.attention(q, k[:5], v[:5], 0.9, k_index=np.arange(5))
    x1 = orc.merge(*orc.merge(a[0], a[1].T, b[0], b[1].T), c[0], c[1].T)
    x2 = orc.merge(a[0], a[1].T, *orc.merge(b[0], b[1].T, c[0], c[1].T))
    np.testing.assert_allclose(x1[0], x2[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(x1[1], x2[1], rtol=1e-13)


# ----------------------------------------------------------------------- ring

def test_ring_order_follows_send_to_next_rank():
    # Simulate the page's loop: at every step each rank sends its KV buffer to
    # rank+1 and receives from rank-1.  The block a rank holds at step t must
    # be ring_block(r, t, P).
    for P in (1, 2, 4, 16):
        held = list(range(P))
        for t in range(P):
            for r in range(P):
                assert orc.ring_block(r, t, P) == held[r]
            held = [held[(r - 1) % P] for r in range(P)]


def test_ring_visits_each_pair_once_and_causal_skip():
    P = 16
    pairs = {(r, orc.ring_block(r, t, P)) for t in range(P) for r in range(P)}
    assert len(pairs) == P * P
    work = sum(len(orc.ring_block_order(r, P)) for r in range(P))
    assert work == P * (P + 1) // 2 == 136
    assert orc.ring_block_order(3, 16) == [3, 2, 1, 0]


def test_ring_ordered_blocks_then_merge_equal_full():
    rng = np.random.default_rng(15)
    N, P = 64, 4
    blk = N // P
    q, k, v = _rand_qkv(rng, N, N, 2, 1, 8)
    full = orc.attention(q, k, v, 0.4)
    O = np.zeros((N, 2, 8))
    L = np.full((2, N), -np.inf)
    for r in range(P):
        rows = np.arange(r * blk, (r + 1) * blk)
        acc_o, acc_l = np.zeros((blk, 2, 8)), np.full((blk, 2), -np.inf)
        for b in orc.ring_block_order(r, P):
            cols = np.arange(b * blk, (b + 1) * blk)
            o, l = orc.attention(q[rows], k[cols], v[cols], 0.4, q_index=rows, k_index=cols)
            acc_o, acc_l = orc.merge(acc_o, acc_l, o, l.T)
        O[rows], L[:, rows] = acc_o, acc_l.T
    np.testing.assert_allclose(O, full[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(L, full[1], rtol=1e-13)


# --------------------------------------------------------------- int8 KV cache

def test_int8_codes_exact_for_representable_rows():
    """Rows k * 2^-e with integer k in [-127, 127] and |k|max = 127: the scale
    is 2^-e exactly, the codes are k and dequantisation gives the row back."""
    rng = np.random.default_rng(40)
    for e in (0, 3, 9):
        k = rng.integers(-127, 128, size=(5, 128))
        k[:, 7] = 127
        k[2, 7] = -127
        x = k.astype(np.float64) * 2.0 ** -e
        codes, scale = orc.quantize_kv_int8(x)
        assert np.array_equal(codes.astype(np.int64), k)
        assert np.all(scale == np.float32(2.0 ** -e))
        assert np.array_equal(orc.dequantize_kv_int8(codes, scale), x)


def test_int8_ties_round_to_even_and_sign_symmetry():
    # amax = 127 -> 127/amax = 1, so code = rint(x): x.5 ties go to the even code
    x = np.array([[127.0, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, 126.5] + [0.0] * 120])
    codes, scale = orc.quantize_kv_int8(x)
    assert scale[0] == np.float32(1.0)
    assert codes[0, :8].tolist() == [127, 2, 4, -2, -4, 0, 2, 126]
    c2, s2 = orc.quantize_kv_int8(-x)
    assert np.array_equal(c2, -codes) and np.array_equal(s2, scale)


def test_int8_zero_row_and_error_bound():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((64, 4, 128)).astype(np.float32) * rng.uniform(1e-3, 50.0, (64, 4, 1)).astype(np.float32)
    x[3, 1] = 0.0
    codes, scale = orc.quantize_kv_int8(x)
    assert scale[3, 1] == 0.0 and not codes[3, 1].any()
    live = scale > 0
    # the largest magnitude of every non-zero row maps to +-127
    assert np.all(np.abs(codes.astype(np.int64)).max(axis=-1)[live] == 127)
    # round-to-nearest: |x - code * scale| <= scale / 2 (plus fp32 rounding of 127/amax)
    err = np.abs(x.astype(np.float64) - orc.dequantize_kv_int8(codes, scale))
    bound = scale.astype(np.float64)[..., None] * (0.5 + 1e-5) + 1e-6 * np.abs(x)
    assert np.all(err <= bound)
    # and the scale is amax / 127
    np.testing.assert_allclose(scale, np.abs(x).max(axis=-1) / 127.0, rtol=1e-7)

"""Float64 CPU oracle for the context-extended attention forward pass.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline / reference arms of ``bench.py`` may
import this module.  The library (``librcx.so`` and its Python binding) never
calls it, and this module imports nothing from the library: the two share no
kernels, helpers, tables or constants.  Inputs reach both sides from the seeded
generators, which hold none of the method's arithmetic.

Everything here is a plain definition in float64 with numpy, written from the
source pages (cited per function as "page title, section"):

  * "Context Extension" concept page (compassingai), sections "RoPE scaling
    schemes" and "Technical principles": RoPE theta_i = base^(-2i/d), the
    rotation R(m) acting on each pair (2i, 2i+1), PI m -> m/s, NTK-aware
    base' = base * s^(d/(d-2)), FlashAttention tiling with a running max.
  * "Context window extension: 4K to 1M" (guijiagi), section 2.1 PI,
    2.2 NTK-aware, 2.3 NTK-by-parts, 2.4 YaRN temperature, 3 dynamic NTK,
    4.1 sliding window, 4.2 StreamingLLM sinks, 5.2-5.3 Ring Attention.
  * kwkr.cn long-context article, section 2.2: ring attention pseudo-code
    (roll the KV chunks by one each step, aggregate online).

Readings taken where the pages are silent, garbled or disagree:
  * rotation pairs are adjacent dimensions (2i, 2i+1), rotated counter-clockwise
    by phi = m * theta_i;
  * NTK-by-parts band edges are L_train/beta (short wavelengths, unscaled) and
    L_train/alpha (long wavelengths, scaled by 1/s), with a ramp linear in the
    wavelength between them that is continuous at both edges;
  * dynamic NTK takes l = L_target as the current sequence length;
  * the sliding window holds w keys, i - w < j <= i; sinks are keys j < n_sink;
  * logits are scaled by 1/(sqrt(d) * t);
  * partial results are combined by an LSE-weighted merge (the page's plain
    "output += block_output" is only right after that weighting);
  * the ring visits, at step t, KV block (r - t) mod P on shard r;
  * an int8 KV cache is symmetric per row of d values: scale = amax / 127 and
    code = rint(x * 127 / amax), decided in IEEE fp32.

Parity pins for every function live in tests/test_oracle_pins.py.
"""

from __future__ import annotations

import math

import numpy as np

# Frequency schedules.  The integer codes are part of the data passed to both
# sides (they name a scheme); they hold no arithmetic.
PLAIN, PI, NTK, DYN_NTK, NTK_PARTS, YARN = 0, 1, 2, 3, 4, 5
SCHEME_NAMES = {PLAIN: "plain", PI: "pi", NTK: "ntk", DYN_NTK: "dyn_ntk",
                NTK_PARTS: "ntk_parts", YARN: "yarn"}


# --------------------------------------------------------------------------
# Frequencies
# --------------------------------------------------------------------------

def rope_theta(base: float, d: int) -> np.ndarray:
    """theta_i = base^(-2i/d) for i = 0 .. d/2-1.

    "Context Extension" concept page, "RoPE scaling schemes" and "Technical
    principles" (RoPE definition); the same exponents appear as
    arange(0, d, 2)/d in "Context window extension: 4K to 1M" section 2.3.
    """
    if d <= 0 or d % 2:
        raise ValueError("head dimension d must be positive and even")
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d)


def ntk_base(base: float, d: int, s: float) -> float:
    """NTK-aware base' = base * s^(d/(d-2)).

    "Context window extension: 4K to 1M" section 2.2; "Context Extension"
    concept page, NTK-aware row of the scheme table.
    """
    return float(base) * float(s) ** (d / (d - 2.0))


def dynamic_ntk_base(base: float, d: int, seq_len: int, L_train: int) -> float:
    """Dynamic NTK: b'(l) = b * (l/L_train)^(d/(d-2)) when l > L_train, else b.

    "Context window extension: 4K to 1M" section 3 (formula and the
    DynamicNTKScaling class: factor 1.0 when seq_len <= train_len).
    """
    if seq_len <= L_train:
        return float(base)
    s = seq_len / L_train
    return float(base) * s ** (d / (d - 2.0))


def ntk_parts_factor(wavelength: float, L_train: float, s: float,
                     alpha: float, beta: float) -> float:
    """Per-pair frequency factor of NTK-by-parts, as a function of wavelength.

    "Context window extension: 4K to 1M" section 2.3: wavelengths much shorter
    than the context are not interpolated, much longer ones are linearly
    interpolated (factor 1/s), with a smooth transition between.  Band edges
    lam_lo = L_train/beta and lam_hi = L_train/alpha; between them the factor
    goes linearly in the wavelength from 1 (at lam_lo) to 1/s (at lam_hi),
    using the page's ramp variable t = (lam_hi - lam)/(lam_hi - lam_lo).
    """
    lam_lo = L_train / beta
    lam_hi = L_train / alpha
    if wavelength < lam_lo:
        return 1.0
    if wavelength > lam_hi:
        return 1.0 / s
    t = (lam_hi - wavelength) / (lam_hi - lam_lo)
    return 1.0 / s + (1.0 - 1.0 / s) * t


def yarn_temperature(s: float) -> float:
    """YaRN attention temperature t = 0.1 ln(s) + 1.

    "Context window extension: 4K to 1M" section 2.4.
    """
    return 0.1 * math.log(s) + 1.0


def rope_freqs(scheme: int, base: float, d: int, L_train: int, L_target: int,
               alpha: float = 1.0, beta: float = 32.0):
    """Effective per-pair frequencies theta'_i (float64, length d/2) and t.

    s = L_target / L_train ("Context window extension: 4K to 1M" 2.1-2.2).
    PI rotates position m by (m/s)*theta_i; it is returned here as the
    equivalent frequency theta_i/s (the rotation angle is a product, so the
    two agree up to one rounding; a pin checks this).  DYN_NTK takes
    l = L_target.  t = 1 except for YARN.
    """
    s = L_target / L_train
    theta = rope_theta(base, d)
    t = 1.0
    if scheme == PLAIN:
        out = theta
    elif scheme == PI:
        out = theta / s
    elif scheme == NTK:
        out = rope_theta(ntk_base(base, d, s), d)
    elif scheme == DYN_NTK:
        out = rope_theta(dynamic_ntk_base(base, d, L_target, L_train), d)
    elif scheme in (NTK_PARTS, YARN):
        lam = 2.0 * math.pi / theta
        f = np.array([ntk_parts_factor(x, L_train, s, alpha, beta) for x in lam])
        out = theta * f
        if scheme == YARN:
            t = yarn_temperature(s)
    else:
        raise ValueError(f"unknown scheme {scheme}")
    return np.asarray(out, dtype=np.float64), float(t)


def rope_freqs_per_pair(base: float, d: int, factors) -> np.ndarray:
    """Per-plane rescaled frequencies theta'_i = theta_i / lambda_i.

    "Context window extension: 4K to 1M" section 2.5 (LongRoPE): instead of
    one factor for all frequencies, each 2D rotation plane i gets its own
    scaling factor lambda_i (found by a search that is not part of this
    path); plane i then interpolates positions by its own factor, m -> m /
    lambda_i, i.e. theta_i / lambda_i.  Every lambda_i must be positive.
    """
    lam = np.asarray(factors, dtype=np.float64)
    if lam.shape != (d // 2,) or not np.all(np.isfinite(lam)) or not np.all(lam > 0):
        raise ValueError("need d/2 positive finite factors")
    return rope_theta(base, d) / lam


# --------------------------------------------------------------------------
# Rotation
# --------------------------------------------------------------------------

def rope_rotate(x: np.ndarray, positions, inv_freq: np.ndarray) -> np.ndarray:
    """Apply R(m) to every token of x.

    x: [N, H, d] (any float, computed in float64); positions: [N] integers.
    Pair (2i, 2i+1) at position m turns by phi = m * theta'_i:
        (x, y) -> (x cos phi - y sin phi, x sin phi + y cos phi).
    "Context Extension" concept page, "Technical principles" (R(m) is the
    rotation matrix acting on each pair of dimensions (2i, 2i+1)).
    """
    x = np.asarray(x, dtype=np.float64)
    m = np.asarray(positions, dtype=np.float64)
    phi = m[:, None] * np.asarray(inv_freq, dtype=np.float64)[None, :]   # [N, d/2]
    c = np.cos(phi)[:, None, :]
    sn = np.sin(phi)[:, None, :]
    xe = x[..., 0::2]
    xo = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * sn
    out[..., 1::2] = xe * sn + xo * c
    return out


# --------------------------------------------------------------------------
# Masks
# --------------------------------------------------------------------------

def visible(i, j, window: int, n_sink: int):
    """Mask predicate on global token indices (query i, key j).

    Causal: j <= i (autoregressive attention, "Context Extension" KV-cache
    decode loop).  Sliding window of w keys, i - w < j <= i ("Context window
    extension: 4K to 1M" section 4.1).  StreamingLLM sinks: keys j < n_sink stay
    visible beside the window (same page, section 4.2).  window == 0: no window.
    """
    i = np.asarray(i)
    j = np.asarray(j)
    causal = j <= i
    if window <= 0:
        return causal
    return causal & ((j > i - window) | (j < n_sink))


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def attention(q, k, v, scale: float, window: int = 0, n_sink: int = 0,
              q_index=None, k_index=None, rows=None):
    """Full-softmax attention with an explicit mask, float64.

    q: [Nq, Hq, d]; k, v: [Nk, Hkv, d] (already rotated); Hq = G * Hkv and
    query head h reads KV head h // G (consecutive GQA groups).
    z_ij = scale * q_i . k_j; masked logits are -inf; O_i = sum_j p_ij v_j with
    p = softmax(z_i); lse_i = max_j z_ij + ln sum_j exp(z_ij - max).
    A row with no visible key gets O = 0 and lse = -inf.
    ("Context Extension" concept page, FlashAttention section: S = QK^T,
    P = softmax(S), O = PV.)

    q_index / k_index: global token index of each q / k row (default arange).
    rows: None for every (token, head), or a dict {head: array of q rows} to
    evaluate only those rows.  Returns (O, lse): full arrays [Nq, Hq, d] /
    [Hq, Nq] when rows is None, else dicts keyed by head.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Nq, Hq, d = q.shape
    Nk, Hkv, _ = k.shape
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    qi = np.arange(Nq) if q_index is None else np.asarray(q_index)
    kj = np.arange(Nk) if k_index is None else np.asarray(k_index)
    heads = range(Hq) if rows is None else rows.keys()
    outs, lses = {}, {}
    for h in heads:
        sel = np.arange(Nq) if rows is None else np.asarray(rows[h])
        g = h // G
        z = (q[sel, h, :] @ k[:, g, :].T) * scale
        mask = visible(qi[sel][:, None], kj[None, :], window, n_sink)
        z = np.where(mask, z, -np.inf)
        mx = z.max(axis=1, initial=-np.inf)
        any_vis = np.isfinite(mx)
        mx_safe = np.where(any_vis, mx, 0.0)
        p = np.exp(z - mx_safe[:, None])            # exp(-inf) = 0 for masked
        l = p.sum(axis=1)
        o = np.zeros((len(sel), d))
        o[any_vis] = (p[any_vis] @ v[:, g, :]) / l[any_vis, None]
        lse = np.full(len(sel), -np.inf)
        lse[any_vis] = mx[any_vis] + np.log(l[any_vis])
        outs[h], lses[h] = o, lse
    if rows is not None:
        return outs, lses
    O = np.stack([outs[h] for h in range(Hq)], axis=1)
    L = np.stack([lses[h] for h in range(Hq)], axis=0)
    return O, L


def attention_blockwise(q, k, v, scale: float, window: int, n_sink: int,
                        block_order, q_index=None, k_index=None):
    """Blockwise attention with an online softmax, visiting KV blocks in order.

    This is the method itself (not the definition): per row keep a running
    max m, running sum l and an unnormalised accumulator; for each KV block
    take m_new = max(m, rowmax z), rescale l and the accumulator by
    exp(m - m_new), add exp(z - m_new) and its product with V.
    ("Context Extension" concept page, FlashAttention section: blocks of
    B_r x B_c, running-max accumulation, no n x n matrix kept.)
    block_order: a list of arrays of key rows, one per visited block.
    Returns (O [Nq, Hq, d], lse [Hq, Nq]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Nq, Hq, d = q.shape
    Nk, Hkv, _ = k.shape
    G = Hq // Hkv
    qi = np.arange(Nq) if q_index is None else np.asarray(q_index)
    kj = np.arange(Nk) if k_index is None else np.asarray(k_index)
    O = np.zeros((Nq, Hq, d))
    LSE = np.full((Hq, Nq), -np.inf)
    for h in range(Hq):
        g = h // G
        m = np.full(Nq, -np.inf)
        l = np.zeros(Nq)
        acc = np.zeros((Nq, d))
        for blk in block_order:
            blk = np.asarray(blk)
            if blk.size == 0:
                continue
            z = (q[:, h, :] @ k[blk, g, :].T) * scale
            z = np.where(visible(qi[:, None], kj[blk][None, :], window, n_sink), z, -np.inf)
            m_new = np.maximum(m, z.max(axis=1))
            live = np.isfinite(m_new)
            m_ref = np.where(live, m_new, 0.0)
            alpha = np.where(np.isfinite(m), np.exp(m - m_ref), 0.0)
            p = np.exp(z - m_ref[:, None])
            l = l * alpha + p.sum(axis=1)
            acc = acc * alpha[:, None] + p @ v[blk, g, :]
            m = m_new
        live = l > 0
        O[live, h, :] = acc[live] / l[live, None]
        LSE[h, live] = m[live] + np.log(l[live])
    return O, LSE


def merge(o_a, lse_a, o_b, lse_b):
    """LSE-weighted merge of two partial attention results over disjoint keys.

    The Ring Attention loop of "Context window extension: 4K to 1M" section 5.3
    adds each block's output into the running output, and the kwkr.cn article
    section 2.2 aggregates the blocks online; for softmax outputs that sum is
    only right with the weights w = exp(lse - m):
        m = max(lse_a, lse_b), o = (w_a o_a + w_b o_b)/(w_a + w_b),
        lse = m + ln(w_a + w_b).  Two empty partials give o = 0, lse = -inf.
    o_*: [..., d]; lse_*: [...] (same leading shape).
    """
    o_a = np.asarray(o_a, dtype=np.float64)
    o_b = np.asarray(o_b, dtype=np.float64)
    lse_a = np.asarray(lse_a, dtype=np.float64)
    lse_b = np.asarray(lse_b, dtype=np.float64)
    m = np.maximum(lse_a, lse_b)
    live = np.isfinite(m)
    m_ref = np.where(live, m, 0.0)
    w_a = np.where(np.isfinite(lse_a), np.exp(lse_a - m_ref), 0.0)
    w_b = np.where(np.isfinite(lse_b), np.exp(lse_b - m_ref), 0.0)
    den = w_a + w_b
    safe = np.where(live, den, 1.0)
    o = np.where(live[..., None], (w_a[..., None] * o_a + w_b[..., None] * o_b) / safe[..., None], 0.0)
    lse = np.where(live, m_ref + np.log(safe), -np.inf)
    return o, lse


# --------------------------------------------------------------------------
# Int8 KV cache
# --------------------------------------------------------------------------

def quantize_kv_int8(x):
    """Symmetric int8 codes and one fp32 scale per (..., row) of a KV cache.

    "Context window extension: 4K to 1M" section 6.1 stores the KV cache in
    INT8 instead of 16-bit floats to halve its memory (the "Context Extension"
    concept page lists the same compression in its KV-cache table).  The pages
    fix no format; the reading taken is the plainest symmetric one, per row of
    d values (one token of one KV head):
        amax = max |x|,  scale = amax / 127,  code = rint(x * (127 / amax)),
    clamped to [-127, 127] (all zero when amax = 0).  The codes are integers
    decided by floating point, so they are computed in IEEE fp32 (division,
    product, round-half-to-even), the precision the device uses too.
    x: [..., d] (the values the device sees); returns (codes int8 [..., d],
    scale float32 [...]).
    """
    xf = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(xf), axis=-1).astype(np.float32)
    live = amax > 0
    safe = np.where(live, amax, np.float32(1)).astype(np.float32)
    scale = np.where(live, safe / np.float32(127), np.float32(0)).astype(np.float32)
    inv = np.where(live, np.float32(127) / safe, np.float32(0)).astype(np.float32)
    prod = (xf * inv[..., None]).astype(np.float32)
    codes = np.clip(np.rint(prod), -127, 127).astype(np.int8)
    return codes, scale


def dequantize_kv_int8(codes, scale):
    """The cache values an int8 KV cache stands for: code * scale (float64)."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scale, dtype=np.float64)[..., None]


# --------------------------------------------------------------------------
# Ring order
# --------------------------------------------------------------------------

def ring_block(r: int, t: int, P: int) -> int:
    """KV block held by shard r at ring step t: (r - t) mod P.

    "Context window extension: 4K to 1M" section 5.3 (each step sends the KV
    buffer to rank+1 and receives from rank-1) and kwkr.cn section 2.2
    (roll the chunks by one per step).  The section 5.2 timeline, which shows
    block r + t, disagrees with both and is taken as garbled.
    """
    return (r - t) % P


def ring_block_order(shard: int, P: int, causal: bool = True):
    """Blocks visited by one shard over steps t = 0..P-1; causal drops b > r."""
    order = [ring_block(shard, t, P) for t in range(P)]
    if causal:
        order = [b for b in order if b <= shard]
    return order


def causal_visible_pairs(N: int, window: int = 0, n_sink: int = 0) -> int:
    """Count of visible (i, j) pairs of an N-token sequence, by enumeration
    over rows (O(N) integer work).  Useful-FLOP counts are 4 * d * Hq * this."""
    total = 0
    for i in range(N):
        if window <= 0:
            total += i + 1
            continue
        lo = max(0, i - window + 1)             # window keys lo..i
        total += i - lo + 1
        total += min(n_sink, lo)                # sinks below the window
    return total

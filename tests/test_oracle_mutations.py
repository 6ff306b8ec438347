"""Mutation check of the oracle's pins: each plausible mistake (a dropped term,
a wrong sign, index, exponent, band edge, window boundary, GQA mapping, ring
direction, merge weight) is planted in a copy of the oracle, on the CPU, and
at least one pin in tests/test_oracle_pins.py must fail on it."""

import importlib.util
import itertools
import os
import sys
import types

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "rcx_oracle.py")

MUTATIONS = [
    ("out[..., 0::2] = xe * c - xo * sn", "out[..., 0::2] = xe * c + xo * sn"),
    ("out[..., 1::2] = xe * sn + xo * c", "out[..., 1::2] = -xe * sn + xo * c"),
    ("return np.power(float(base), -2.0 * i / d)", "return np.power(float(base), -1.0 * i / d)"),
    ("float(s) ** (d / (d - 2.0))", "float(s) ** (d / (d - 1.0))"),
    ("return 1.0 / s + (1.0 - 1.0 / s) * t", "return 1.0 - (1.0 - 1.0 / s) * t"),
    ("lam_lo = L_train / beta", "lam_lo = L_train / (2 * math.pi) * beta"),
    ("return 0.1 * math.log(s) + 1.0", "return 0.1 * math.log(s) + 1.1"),
    ("return causal & ((j > i - window) | (j < n_sink))", "return causal & ((j >= i - window) | (j < n_sink))"),
    ("return causal & ((j > i - window) | (j < n_sink))", "return causal & ((j > i - window) | (j <= n_sink))"),
    ("causal = j <= i", "causal = j < i"),
    ("g = h // G\n        z = (q[sel, h, :]", "g = h % Hkv\n        z = (q[sel, h, :]"),
    ("lse[any_vis] = mx[any_vis] + np.log(l[any_vis])", "lse[any_vis] = np.log(l[any_vis])"),
    ("return (r - t) % P", "return (r + t) % P"),
    ("(w_a[..., None] * o_a + w_b[..., None] * o_b) / safe[..., None]", "(w_a[..., None] * o_a + w_b[..., None] * o_b)"),
    ("acc = acc * alpha[:, None] + p @ v[blk, g, :]", "acc = acc + p @ v[blk, g, :]"),
    ("out = theta / s", "out = theta * s"),
    ("s = seq_len / L_train", "s = L_train / seq_len"),
    ("total += min(n_sink, lo)", "total += n_sink"),
    ("return rope_theta(base, d) / lam", "return rope_theta(base, d) * lam"),
    ("scale = np.where(live, safe / np.float32(127), np.float32(0))", "scale = np.where(live, safe / np.float32(128), np.float32(0))"),
    ("codes = np.clip(np.rint(prod), -127, 127)", "codes = np.clip(np.floor(prod + 0.5), -127, 127)"),
    ("codes = np.clip(np.rint(prod), -127, 127)", "codes = np.clip(np.trunc(prod), -127, 127)"),
    ("inv = np.where(live, np.float32(127) / safe, np.float32(0))", "inv = np.where(live, np.float32(127.5) / safe, np.float32(0))"),
]


def _load_mutant(src_text):
    mod = types.ModuleType("oracle.rcx_oracle")
    mod.__file__ = SRC
    exec(compile(src_text, SRC, "exec"), mod.__dict__)
    return mod


def _pin_module(oracle_mod):
    import oracle
    saved = sys.modules.get("oracle.rcx_oracle")
    sys.modules["oracle.rcx_oracle"] = oracle_mod
    old_attr = getattr(oracle, "rcx_oracle", None)
    oracle.rcx_oracle = oracle_mod
    try:
        spec = importlib.util.spec_from_file_location("_pins_under_test", os.path.join(HERE, "test_oracle_pins.py"))
        m = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(m)
    finally:
        if saved is not None:
            sys.modules["oracle.rcx_oracle"] = saved
        if old_attr is not None:
            oracle.rcx_oracle = old_attr
    return m


def _cases(fn):
    """Expand pytest.mark.parametrize marks into keyword dicts."""
    grids = []
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names, values = mark.args[0], mark.args[1]
        names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
        grids.append([dict(zip(names, v if len(names) > 1 else (v,))) for v in values])
    if not grids:
        return [{}]
    out = []
    for combo in itertools.product(*grids):
        d = {}
        for part in combo:
            d.update(part)
        out.append(d)
    return out


def _some_pin_fails(pins):
    for name in dir(pins):
        if not name.startswith("test_"):
            continue
        fn = getattr(pins, name)
        for kw in _cases(fn):
            try:
                fn(**kw)
            except Exception:
                return True
    return False


def test_unmutated_oracle_passes_every_pin():
    src = open(SRC).read()
    assert not _some_pin_fails(_pin_module(_load_mutant(src)))


@pytest.mark.parametrize("i", range(len(MUTATIONS)))
def test_planted_mistake_is_caught(i):
    old, new = MUTATIONS[i]
    src = open(SRC).read()
    assert old in src, old
    mutant = _load_mutant(src.replace(old, new, 1))
    assert _some_pin_fails(_pin_module(mutant)), f"no pin catches: {new!r}"

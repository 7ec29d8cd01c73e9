"""Mutation check of the oracle's pins: each case plants one plausible slip in
an in-memory copy of the oracle's source (the file itself is never touched),
runs the pins of tests/test_oracle_pins.py against that copy, and requires at
least one of them to fail. A slip that every pin let through would mean that
part of the oracle is pinned only by itself."""
import importlib.util
import inspect
import os
import types

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE = os.path.join(os.path.dirname(HERE), "oracle", "vggt_oracle.py")

# (name, original source fragment, planted slip); each fragment occurs once
MUTATIONS = [
    ("score scale dropped",
     "scores = (qh @ kh.T) / math.sqrt(qh.shape[-1])", "scores = (qh @ kh.T)"),
    ("softmax not normalised",
     "return e / np.sum(e, axis=axis, keepdims=True)", "return e"),
    ("unbiased variance",
     "var = (c * c).mean(axis=-1, keepdims=True)",
     "var = (c * c).sum(axis=-1, keepdims=True) / (x.shape[-1] - 1)"),
    ("LayerNorm eps missing",
     "y = c / np.sqrt(var + eps)", "y = c / np.sqrt(var)"),
    ("LayerNorm not centred",
     "c = x - mu", "c = x"),
    ("affine shift before the scale",
     "        y = y * np.asarray(gamma, dtype=np.float64)",
     "        y = (y + 1.0) * np.asarray(gamma, dtype=np.float64) - 1.0"),
    ("RoPE sign",
     "= x1 * c - x2 * s", "= x1 * c + x2 * s"),
    ("RoPE row and column halves swapped",
     "theta = pos[..., a][..., None] * freq", "theta = pos[..., 1 - a][..., None] * freq"),
    ("RoPE frequency exponent",
     "return base ** (-2.0 * i / d)", "return base ** (-1.0 * i / d)"),
    ("pool members column-major",
     "cells.append([r * gw + c for r in rows for c in cols])",
     "cells.append([r * gw + c for c in cols for r in rows])"),
    ("pool edge cells not clipped",
     "rows = range(cr * kd, min(cr * kd + kd, gh))", "rows = range(cr * kd, cr * kd + kd)"),
    ("pooled position of the first member",
     "pp[:, i] = pos[:, idx].mean(axis=1)", "pp[:, i] = pos[:, idx[0]]"),
    ("frame key range one short",
     "lo, hi = s * T, (s + 1) * T", "lo, hi = s * T, (s + 1) * T - 1"),
    ("bf16 rounding truncates",
     "rounded = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)", "rounded = (u >> 16).astype(np.uint16)"),
]


def _load_pins():
    spec = importlib.util.spec_from_file_location("oracle_pins_under_mutation", os.path.join(HERE, "test_oracle_pins.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _pin_calls(pins):
    """Every pin as a zero-argument call (parametrized pins once per case)."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_") or fn.__module__ != pins.__name__:
            continue
        params = list(inspect.signature(fn).parameters)
        if not params:
            calls.append((name, fn, {}))
            continue
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            names = [n.strip() for n in mark.args[0].split(",")] if isinstance(mark.args[0], str) else list(mark.args[0])
            for values in mark.args[1]:
                values = values if len(names) > 1 else (values,)
                calls.append((name, fn, dict(zip(names, values))))
    return calls


def _mutant(src: str, old: str, new: str):
    assert src.count(old) == 1, old
    mod = types.ModuleType("vggt_oracle_mutant")
    mod.__file__ = ORACLE
    exec(compile(src.replace(old, new), ORACLE + " (mutant)", "exec"), mod.__dict__)
    return mod


def test_pins_pass_on_the_oracle_itself():
    pins = _load_pins()
    for name, fn, kw in _pin_calls(pins):
        fn(**kw)


@pytest.mark.parametrize("what,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_every_planted_slip_fails_a_pin(what, old, new):
    src = open(ORACLE, encoding="utf-8").read()
    pins = _load_pins()
    pins.O = _mutant(src, old, new)
    caught = None
    for name, fn, kw in _pin_calls(pins):
        try:
            fn(**kw)
        except Exception:  # an assertion, or the slip breaking the pin's arithmetic
            caught = name
            break
    assert caught is not None, f"no pin fails when the oracle has: {what}"

"""The oracle's pins are not vacuous: plausible mistakes planted in copies of the
oracle (on the CPU) are each rejected by at least one pin.

Every mutant below is a one-line edit of the oracle's source (a dropped term, a
wrong sign, a transposed operand, a wrong rounding or bit order, ...).  The pins
of ``test_oracle_pins.py`` -- closed forms, brute force, worked examples and
invariants, none of which re-derives the oracle's own formulas -- run against
the mutant with the oracle package's functions replaced, and at least one of them
must fail.  The planted mistakes live only in these in-memory copies.
"""

import importlib.util
import itertools
import os
import types

import pytest

import oracle
import test_oracle_pins as pins

SRC_PATH = os.path.join(os.path.dirname(oracle.__file__), "gptq_ref.py")

# (name, exact source text, replacement)
MUTANTS = [
    ("Hessian without the factor 2", "    return 2.0 * H\n", "    return H\n"),
    ("damping from the diagonal's sum", "lam = float(damp) * float(np.mean(np.diag(H)))",
     "lam = float(damp) * float(np.sum(np.diag(H)))"),
    ("act-order ascending", "return np.argsort(-np.diag(np.asarray(H, dtype=F64)), kind=\"stable\")",
     "return np.argsort(np.diag(np.asarray(H, dtype=F64)), kind=\"stable\")"),
    ("lower factor returned for U", "    return np.ascontiguousarray(L.T)\n",
     "    return np.ascontiguousarray(L)\n"),
    ("Cholesky of H_d instead of its inverse", "    Hinv = np.linalg.inv(np.asarray(Hd, dtype=F64))\n",
     "    Hinv = np.asarray(Hd, dtype=F64)\n"),
    ("range not widened to include 0", "    xmin = np.minimum(x.min(axis=1), 0.0)\n",
     "    xmin = x.min(axis=1)\n"),
    ("zero point truncated", "    z = np.rint(-xmin / s)\n", "    z = np.floor(-xmin / s)\n"),
    ("ties rounded away from zero",
     "    return np.clip(np.rint(np.asarray(w, dtype=F64) / s) + z, 0, maxq)\n",
     "    return np.clip(np.floor(np.asarray(w, dtype=F64) / s + 0.5) + z, 0, maxq)\n"),
    ("dequantisation without the zero point", "    return s * (q - z)\n", "    return s * q\n"),
    ("error not divided by U_jj", "            e = (w - wq) / U[j, j]\n",
     "            e = (w - wq)\n"),
    ("compensation with the wrong sign",
     "                W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])\n",
     "                W[:, j + 1:b1] += np.outer(e, U[j, j + 1:b1])\n"),
    ("deferred update with a transposed block of U",
     "            W[:, b1:] -= E[:, b0:b1] @ U[b0:b1, b1:]\n",
     "            W[:, b1:] -= E[:, b0:b1] @ U[b1:, b0:b1].T\n"),
    ("deferred update dropped", "            W[:, b1:] -= E[:, b0:b1] @ U[b0:b1, b1:]\n",
     "            pass\n"),
    ("group parameters from the original weights",
     "                s, z = quant_params(W[:, j:j + group], bits, sym)\n",
     "                s, z = quant_params(W0[:, j:j + group], bits, sym)\n"),
    ("symmetric scale over 2^b - 1", "amax / (half - 1))", "amax / (2 * half - 1))"),
    ("symmetric zero point stored as 0", "return s, np.full_like(s, float(half))",
     "return s, np.zeros_like(s)"),
    ("symmetric range from the signed maximum", "amax = np.abs(x).max(axis=1)",
     "amax = x.max(axis=1)"),
    ("static groups ignored", "    if static_groups and group != -1:\n", "    if False:\n"),
    ("static groups indexed by sweep position", "fixed = (fs, fz, perm // group)",
     "fixed = (fs, fz, np.arange(d) // group)"),
    ("static parameters from the permuted weights",
     "quant_params(W[:, k * group:(k + 1) * group], bits, sym)",
     "quant_params(W[:, perm][:, k * group:(k + 1) * group], bits, sym)"),
    ("chain inputs not propagated", "        X = (X.astype(F64) @ Wh16.T).astype(np.float16)\n",
     "        pass\n"),
    ("chain run on the original weights", "        Wh16 = out[\"What\"].astype(np.float16).astype(F64)\n",
     "        Wh16 = np.asarray(W, dtype=F64).astype(np.float16).astype(F64)\n"),
    ("chain outputs kept in float64", "        X = (X.astype(F64) @ Wh16.T).astype(np.float16)\n",
     "        X = X.astype(F64) @ Wh16.T\n"),
    ("chain weights not rounded to fp16", "        Wh16 = out[\"What\"].astype(np.float16).astype(F64)\n",
     "        Wh16 = out[\"What\"]\n"),
    ("bit stream most-significant first", "        v = codes[:, c].astype(np.uint64) << np.uint64(off)\n",
     "        v = codes[:, c].astype(np.uint64) << np.uint64(32 - bits - off if off + bits <= 32 else off)\n"),
]

# The group-parameter mutant needs the original weights at hand.
_SWEEP_COPY = "    W = np.array(W, dtype=F64, copy=True)\n"
_SWEEP_COPY_W0 = "    W = np.array(W, dtype=F64, copy=True)\n    W0 = W.copy()\n"


def _mutant_module(old: str, new: str) -> types.ModuleType:
    src = open(SRC_PATH).read()
    assert src.count(old) == 1, old
    src = src.replace(old, new)
    if "W0[" in new:
        assert src.count(_SWEEP_COPY) == 1
        src = src.replace(_SWEEP_COPY, _SWEEP_COPY_W0)
    spec = importlib.util.spec_from_loader("oracle_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src, SRC_PATH + " (mutant)", "exec"), mod.__dict__)
    return mod


def _pin_calls():
    """Every pin of test_oracle_pins as (name, zero-argument callable), with its
    parametrisations expanded."""
    calls = []
    for name in sorted(dir(pins)):
        fn = getattr(pins, name)
        if not (name.startswith("test_") and callable(fn)):
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            calls.append((name, fn))
            continue
        axes = []
        for m in marks:
            argnames, values = m.args[0], m.args[1]
            keys = [a.strip() for a in argnames.split(",")]
            axes.append([dict(zip(keys, v if len(keys) > 1 else (v,))) for v in values])
        for combo in itertools.product(*axes):
            kw = {}
            for part in combo:
                kw.update(part)
            calls.append((f"{name}{kw}", lambda fn=fn, kw=kw: fn(**kw)))
    return calls


PIN_CALLS = _pin_calls()


def test_pins_pass_on_the_oracle_itself():
    # The harness runs the pins correctly: unmutated, every one passes.
    for name, call in PIN_CALLS:
        call()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_rejected(monkeypatch, name, old, new):
    mutant = _mutant_module(old, new)
    for attr in dir(oracle):
        if not attr.startswith("_") and hasattr(mutant, attr):
            monkeypatch.setattr(oracle, attr, getattr(mutant, attr))
    caught = []
    for pin, call in PIN_CALLS:
        try:
            call()
        except Exception:   # an assertion, or the mutant breaking a pin outright
            caught.append(pin)
            break
    assert caught, f"no pin rejects the mutant: {name}"

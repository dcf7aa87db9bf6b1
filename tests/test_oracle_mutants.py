"""The oracle's pins must catch plausible mistakes: each planted mistake (a dropped term, a wrong
sign, index or tie rule, a transposed operand, a wrong head map or position) is compiled into a
separate build of the oracle, and at least one pin must fail against it.  CPU only."""
import inspect
import os

import pytest

import oracle as O
from tests import test_oracle_pins as pins

MUTANTS = {
    1: "ReLU dropped from the head sum",
    2: "ties go to the higher block index",
    3: "own block scored as a candidate",
    4: "query's own token left out",
    5: "wrong GQA head map (h % Hkv)",
    6: "pooling drops one key of the block",
    7: "RoPE rotation sign flipped",
    8: "softmax scale missing",
    9: "indexer query operand transposed",
    10: "pooled key rotated at the block end",
    11: "bf16 rounding truncates",
    12: "YaRN ramp reversed (fast pairs interpolated, slow pairs kept)",
    13: "log-sum-exp without the running maximum",
    14: "indexer head weights ignored",
    15: "every sequence scored against the first sequence's pooled keys",
}


def _pin_calls():
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if params:
            argnames = [a.strip() for a in params[0].args[0].split(",")]
            for vals in params[0].args[1]:
                vals = vals if isinstance(vals, tuple) else (vals,)
                calls.append((name, fn, dict(zip(argnames, vals))))
        else:
            calls.append((name, fn, {}))
    return calls


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, tmp_path):
    path = O.build_mutant(mutant, os.path.join(tmp_path, f"libqsa_oracle_m{mutant}.so"))
    O.use_library(path)
    failed = []
    try:
        for name, fn, kw in _pin_calls():
            try:
                fn(**kw)
            except Exception:
                failed.append(name)
    finally:
        O.use_library(None)
    assert failed, f"no pin caught mutant {mutant}: {MUTANTS[mutant]}"

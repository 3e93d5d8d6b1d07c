"""The oracle's pins reject planted mistakes (oracle/mutation_check.py).

Every mutant's text must still occur exactly once in the oracle's source, so
that the check keeps planting what it names; a few mutants from different
parts of the oracle (the update, the layout, the overflow rule) are built
and run against the pin tests here. The full list runs as
`python oracle/mutation_check.py`.
"""
import os
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "oracle"))
import mutation_check as M  # noqa: E402


def test_every_mutant_still_applies():
    src = open(M.SRC).read()
    stale = [name for name, old, _ in M.MUTANTS if src.count(old) != 1]
    assert not stale, stale
    assert len({name for name, _, _ in M.MUTANTS}) == len(M.MUTANTS)


@pytest.mark.parametrize("name", ["update_sign", "shard_rounding", "overflow_misses_inf"])
def test_pins_reject_a_planted_mistake(name):
    (old, new), = [(o, n) for k, o, n in M.MUTANTS if k == name]
    with tempfile.TemporaryDirectory() as tmp:
        verdict, detail = M.run_one(name, old, new, tmp)
    assert verdict == "caught", detail

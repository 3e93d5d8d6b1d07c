"""The oracle's pins from C (tests/c_oracle_pins.c): a strict C99 program,
linked to the oracle alone, checks it against the golden fixtures (the
hand-computed AdamW steps, the pages' memory figures, the hand-written
loss-scale sequences, the worked layouts), and a planted mistake in the
oracle makes it fail."""
import os
import subprocess
import tempfile

import pytest

import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
GOLDEN = [os.path.join(HERE, "golden", f)
          for f in ("adamw_one_param.txt", "memory_pages.txt", "fsm_sequences.txt", "layout_worked.txt")]


def _build(tmp, lib):
    exe = os.path.join(tmp, "c_oracle_pins")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-O1",
                    "-I", os.path.join(ROOT, "oracle"), os.path.join(HERE, "c_oracle_pins.c"),
                    lib, "-lm", "-o", exe, "-Wl,-rpath," + os.path.dirname(lib)], check=True)
    return exe


def test_c_program_passes_on_the_oracle():
    lib = O.lib()._name
    with tempfile.TemporaryDirectory() as tmp:
        r = subprocess.run([_build(tmp, lib), *GOLDEN], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "oracle pins ok" in r.stdout


@pytest.mark.parametrize("old,new,where", [
    ("st->scale = st->scale * st->growth_factor;", "st->scale = st->scale * 4.0f;", "fsm"),
    ("int64_t S = round_up((L + R - 1) / R, 8);", "int64_t S = round_up(L / R, 8);", "layout"),
    ("float pp = *p * c->dec;", "float pp = *p;", "adamw"),
])
def test_c_program_catches_a_planted_mistake(old, new, where):
    # the same program against an oracle with one planted mistake
    src = open(os.path.join(ROOT, "oracle", "zero_oracle.c")).read()
    assert src.count(old) == 1
    bad = src.replace(old, new)
    with tempfile.TemporaryDirectory() as tmp:
        c = os.path.join(tmp, "zero_oracle.c")
        open(c, "w").write(bad)
        lib = os.path.join(tmp, "liboracle_mutant.so")
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                        "-I", os.path.join(ROOT, "oracle"), c, "-o", lib, "-lm"], check=True)
        r = subprocess.run([_build(tmp, lib), *GOLDEN], capture_output=True, text=True)
    assert r.returncode == 1 and ("FAIL " + where) in r.stderr

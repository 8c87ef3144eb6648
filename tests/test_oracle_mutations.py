"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in the oracle (tests/oracle_mutants.py) and runs
tests/test_oracle_pins.py in a child pytest process: at least one pin must fail. A control
run with nothing planted must pass, so a failing child means the pins, not the harness.
"""
import os
import subprocess
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from oracle_mutants import MUTANTS  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_pins(mutant: str) -> subprocess.CompletedProcess:
    env = dict(os.environ, AWQ_ORACLE_MUTANT=mutant)
    return subprocess.run(
        [sys.executable, "-m", "pytest", os.path.join("tests", "test_oracle_pins.py"), "-q",
         "-x", "-m", "not gpu", "-p", "no:cacheprovider"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_pins_pass_with_nothing_planted():
    r = _run_pins("none")
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_planted_mistake(mutant):
    r = _run_pins(mutant)
    assert r.returncode == 1, f"no pin fails with the oracle mutant {mutant!r}:\n{r.stdout[-2000:]}"

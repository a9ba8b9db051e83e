"""The oracle's pins catch plausible mistakes: each mutant of tests/oracle_mutants.py (one
planted mistake in the CPU oracle) is applied in a child process, and the pins of
tests/test_oracle_pins.py must then fail.  The unmutated oracle passes the same pins (they
run in the suite as usual), so a failure here is the mutant's.
"""
import os
import subprocess
import sys

import pytest

from oracle_mutants import MUTANTS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.join(ROOT, "tests")

_CHILD = (
    "import sys; sys.path[:0] = [{root!r}, {tests!r}]\n"
    "import oracle_mutants\n"
    "oracle_mutants.apply({name!r})\n"
    "import pytest\n"
    "sys.exit(pytest.main(['-q', '-x', '-p', 'no:cacheprovider', '-p', 'no:randomly',\n"
    "                      '-m', 'not gpu', {pins!r}]))\n")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_the_mutant(name):
    code = _CHILD.format(root=ROOT, tests=TESTS, name=name,
                         pins=os.path.join(TESTS, "test_oracle_pins.py"))
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    # pytest exit code 1: some pin failed (the mutant was caught); 0: every pin passed
    assert r.returncode == 1, (f"mutant {name!r} (exit {r.returncode}) survived the pins:\n"
                               f"{r.stdout[-3000:]}\n{r.stderr[-2000:]}")

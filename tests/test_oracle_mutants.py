"""The oracle's pins catch plausible mistakes planted in the oracle (CPU only).

Each mutant of ``oracle_mutants.py`` replaces one oracle function with a copy carrying one
mistake (a dropped scale or term, a reversed sign, a swapped axis, index or operand, an
off-by-one in the cache or the time ids, a wrong rounding rule). The oracle's pin tests run
in a child pytest with that mutant planted; every mutant must make at least one pin fail.
The unmutated pins are the ordinary ``test_oracle_*.py`` run of this suite.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

from oracle_mutants import MUTANTS

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
PINS = ["test_oracle_attention.py", "test_oracle_bf16_flow.py", "test_oracle_cache_rope.py",
        "test_oracle_cross.py", "test_oracle_rope_slots.py"]


def _run_pins(mutant):
    env = dict(os.environ, RKV_ORACLE_MUTANT=mutant,
               PYTHONPATH=os.pathsep.join([ROOT, HERE, os.environ.get("PYTHONPATH", "")]))
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-p", "oracle_mutants",
           *[os.path.join(HERE, f) for f in PINS]]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    return mutant, r.returncode, r.stdout[-1500:]


@pytest.fixture(scope="module")
def outcomes():
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        return {m: (rc, out) for m, rc, out in ex.map(_run_pins, sorted(MUTANTS))}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_planted_mistake(mutant, outcomes):
    rc, out = outcomes[mutant]
    # pytest exit code 1: tests ran and at least one failed (2-5 would be a broken run)
    assert rc == 1, f"mutant {mutant} survived the pins (exit {rc}):\n{out}"


def test_unmutated_pins_pass_under_the_plugin():
    _, rc, out = _run_pins("")
    assert rc == 0, out

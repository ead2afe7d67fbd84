"""The oracle's pins catch plausible mistakes.

Every entry of tests/oracle_mutants.py plants one mistake in one oracle
module (on the CPU, in a child pytest process) and runs that module's pin
file: some pin must fail (pytest exit status 1).  A mistake the pins let
through is a gap in the pins.
"""

import importlib
import inspect
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

from oracle_mutants import MUTANTS

HERE = os.path.dirname(os.path.abspath(__file__))


def _run(k):
    name, modname, old, new, pin_file = MUTANTS[k]
    env = dict(os.environ, VELOX_ORACLE_MUTANT=str(k), CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu", os.path.join(HERE, pin_file)],
                       env=env, capture_output=True, text=True, timeout=900, cwd=HERE)
    return k, r.returncode, r.stdout[-1500:] + r.stderr[-500:]


def test_every_mutant_applies():
    for name, modname, old, new, _ in MUTANTS:
        src = inspect.getsource(importlib.import_module(modname))
        assert src.count(old) == 1, f"{name}: text found {src.count(old)} times"
        assert old != new, name


def test_pins_catch_every_planted_mistake():
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(_run, range(len(MUTANTS))))
    survivors = [(MUTANTS[k][0], rc, out) for k, rc, out in results if rc != 1]
    assert not survivors, "pins did not fail for:\n" + "\n".join(
        f"- {name} (exit {rc})\n{out}" for name, rc, out in survivors)

"""The oracle's pins catch plausible mistakes.

For every planted mistake in tests/oracle_mutants.py, the oracle's pin files
run in a child process with that one oracle function replaced, and the run
must fail; with no mistake planted ("none") the same run must pass, so a
failure is the pins' doing and not the harness's.  Everything runs on the
CPU.  The scale-layout index function is not among the mutants: it is a
storage order, not arithmetic, and a wrong one is caught on the GPU (the
tensor core would read the scales elsewhere and Y would differ).
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

from tests import oracle_mutants

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = ["tests/test_oracle_mxfp4.py", "tests/test_oracle_path.py", "tests/test_oracle_gelu.py"]


def _run_pins(mutant: str) -> subprocess.CompletedProcess:
    env = dict(os.environ, W4A4_ORACLE_MUTANT=mutant)
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           "-p", "tests.oracle_mutants", "-m", "not gpu", *PINS]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_pins_pass_with_nothing_planted():
    r = _run_pins("none")
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


def test_pins_catch_every_planted_mistake():
    # one child per mutant, several at a time (each spends most of its few
    # seconds importing); exit code 1 = tests failed (an exception in a test
    # counts as a failure), anything else would mean the harness broke
    names = sorted(oracle_mutants.MUTANTS)
    workers = max(2, min(8, os.cpu_count() or 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        results = dict(zip(names, ex.map(_run_pins, names)))
    missed = {n: r.returncode for n, r in results.items() if r.returncode != 1}
    assert not missed, "pins passed or the run broke: " + ", ".join(
        f"{n} (rc {rc})" for n, rc in missed.items()) + "\n" + \
        "\n".join(results[n].stdout[-1500:] for n in missed)

"""Pin strength: every planted mistake in tests/oracle_mutants.py must make at least one
oracle pin in tests/test_oracle.py fail (CPU only).

Each mutant runs the pins in a fresh interpreter with one oracle function replaced.
The golden regression record is left out of those runs, since the oracle wrote it
itself; a mistake counts as caught only when an independent pin (a library routine,
a closed form, brute force, an invariant, a planted result) fails.  A run with no
mutant must pass, so the failures come from the mistakes and not from the harness.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

from tests.oracle_mutants import MUTANTS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
RUNNER = (
    "import sys\n"
    "sys.path.insert(0, sys.argv[2])\n"
    "from tests import oracle_mutants\n"
    "oracle_mutants.apply(sys.argv[1])\n"
    "import pytest\n"
    "sys.exit(pytest.main(['-x', '-q', '-p', 'no:cacheprovider', '-m', 'not gpu',\n"
    "                      '--deselect', 'tests/test_oracle.py::test_golden_tiny_regression',\n"
    "                      'tests/test_oracle.py']))\n"
)


def run_pins(name):
    env = dict(os.environ, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-c", RUNNER, name, ROOT], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    failed = [ln.split()[1] for ln in r.stdout.splitlines() if ln.startswith("FAILED ")]
    return name, r.returncode, failed, r.stdout[-2000:] + r.stderr[-2000:]


def test_every_planted_mistake_fails_a_pin():
    names = ["none"] + list(MUTANTS)
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = {name: (rc, failed, tail) for name, rc, failed, tail in ex.map(run_pins, names)}
    rc, _, tail = results.pop("none")
    assert rc == 0, "the pins fail without any mutant:\n" + tail
    survivors = [n for n, (rc, _, _) in results.items() if rc == 0]
    broken = {n: tail for n, (rc, _, tail) in results.items() if rc not in (0, 1)}
    assert not broken, f"harness errors (not test failures): {broken}"
    assert not survivors, f"mistakes no pin catches: {survivors}"
    for n, (_, failed, _) in sorted(results.items()):
        print(f"{n:28s} caught by {failed[0] if failed else '?'}")

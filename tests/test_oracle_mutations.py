"""The pins catch planted mistakes (CPU only).

Each case rebuilds the oracle with one deliberate mistake planted
(ORACLE_PLANT_MISTAKE=n, see the C source) and runs the pin file that should
catch it in a child pytest; the child run must FAIL.  This is what shows the
pins are not a retyping of the oracle: a dropped term, a wrong sign, swapped
operands or a wrong tie rule each break at least one of them.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PLANTS = [
    (1, "E2M1/E4M3 ties to the odd code", "tests/test_oracle_mx.py"),
    (2, "scale exponent rule off by one", "tests/test_oracle_mx.py"),
    (3, "top-k ties: highest index wins", "tests/test_oracle_routing.py"),
    (4, "FP4 nibble order swapped", "tests/test_oracle_layer.py"),
    (5, "gate and up halves swapped", "tests/test_oracle_layer.py"),
    (6, "sign error inside silu", "tests/test_oracle_layer.py"),
    (7, "last routed slot dropped", "tests/test_oracle_layer.py"),
    (8, "weights not renormalised", "tests/test_oracle_routing.py"),
    (9, "grouping not stable", "tests/test_oracle_routing.py"),
    (10, "given routing: local expert offset ignored", "tests/test_oracle_routed.py"),
    (11, "shared expert added with weight 1/2", "tests/test_oracle_shared.py"),
]


@pytest.mark.parametrize("plant,what,pin_file", PLANTS, ids=[p[1] for p in PLANTS])
def test_planted_mistake_is_caught(plant, what, pin_file):
    env = dict(os.environ, ORACLE_PLANT_MISTAKE=str(plant))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", pin_file],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, f"planted mistake '{what}' was not caught:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout

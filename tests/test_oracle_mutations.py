"""The pins have teeth: for each mistake planted in the oracle (ORACLE_MUTATION in
oracle/sage_oracle.c: a rounding rule changed, a sign flipped, a term dropped, an
off-by-one), the pin suite run against that oracle fails.  Each mutant runs the pins
in a child process (SAGE_ORACLE_MUTATION selects it) until the first failure."""
import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    1: "E4M3 rounding ties away from zero",
    2: "fp16 rounding truncates",
    3: "E2M1 ties round upward",
    4: "INT8 codes truncate",
    5: "a ragged Q block averages over 128 rows",
    6: "K smoothing adds the mean",
    7: "delta_V = amax * Vr",
    8: "dS sign flipped",
    9: "causal mask off by one",
    10: "the last key of a tile is missed by the running max",
    11: "the 1 / Pr of the output dropped",
    12: "FP4 tile scale g = amax / 6 (no E4M3 headroom for the block scales)",
    13: "an FP4 block scale that underflows E4M3 stays 0",
    14: "the online-softmax rescale factor inverted",
    15: "the causal mask aligned top-left when N_q != N_kv",
    16: "dS formed from the dequantized K instead of the smoothed K",
    17: "a K group's amax misses its last key",
}


def _run_pins(k):
    env = dict(os.environ, SAGE_ORACLE_MUTATION=str(k), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-x",
                        "-q", "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return k, r.returncode, r.stdout[-400:]


def test_every_planted_mistake_fails_a_pin():
    for k in MUTATIONS:   # build the mutants once, before the child processes start
        oracle.build(mutation=k)
    with cf.ThreadPoolExecutor(max_workers=6) as ex:
        results = list(ex.map(_run_pins, MUTATIONS))
    survivors = [(k, MUTATIONS[k], out) for k, rc, out in results if rc == 0]
    assert not survivors, "planted mistakes no pin rejects: %s" % survivors
    # a failure must be a failed pin, not a crash of the run
    for k, rc, out in results:
        assert rc == 1, "mutation %d: pytest exit code %d\n%s" % (k, rc, out)

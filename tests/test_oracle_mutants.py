"""The oracle's pins have teeth: each build below plants one plausible
mistake in the oracle (on the CPU, through the OR_MUTANT hooks of
oracle/fos_oracle.c), and the pin suite tests/test_oracle_pins.py must fail
on it.  A mistake that no pin caught would mean a part of the oracle that
only checks itself.  The mutant runs go in parallel, one process each."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    1: "4/6 choice takes 4 on ties (err4 <= err6)",
    2: "4/6 tensor scale divides by 6*448 instead of 4*448",
    3: "E2M1 rounding breaks ties upward instead of to the even code",
    4: "block error drops its last term",
    5: "residual adds q*e instead of subtracting it",
    6: "E4M3 scale rounds toward zero instead of to nearest",
    7: "RHT signs read from Philox output word 1 instead of word 0",
    8: "SR rounds up when 2*byte+1 equals 512*p (<= instead of <)",
    9: "MXFP4 exponent floor(log2 a) - 1 instead of - 2",
    10: "dequantize leaves out the tensor scale",
    11: "SR reads the byte of the next element",
    15: "the 4-candidate scale maps the block max to 3 instead of 4",
    16: "Philox first key increment off by one",
    17: "bf16 rounding breaks ties upward instead of to even",
    18: "SR Philox counter is the element index instead of index / 16",
    19: "2D transposed copy's choice bit at the source tile's index",
    20: "colwise transform: the colwise amax taken before the transform",
}

PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")


def _run_all(mutants, parallel=8):
    """{k: (returncode, tail of output)} of the pin suite on each mutant."""
    for k in mutants:   # build serially (gcc), run in parallel
        env = dict(os.environ, FOS_ORACLE_MUTANT=str(k))
        subprocess.run([sys.executable, "-c", "import oracle; oracle.build()"], cwd=ROOT, env=env,
                       check=True, timeout=300)
    out, todo, running = {}, list(mutants), []
    while todo or running:
        while todo and len(running) < parallel:
            k = todo.pop(0)
            env = dict(os.environ, FOS_ORACLE_MUTANT=str(k))
            p = subprocess.Popen([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider",
                                  "-m", "not gpu"], cwd=ROOT, env=env, stdout=subprocess.PIPE,
                                 stderr=subprocess.STDOUT, text=True)
            running.append((k, p))
        k, p = running.pop(0)
        text, _ = p.communicate(timeout=600)
        out[k] = (p.returncode, text[-1500:])
    return out


def test_pins_catch_every_planted_mistake():
    res = _run_all(sorted(MUTANTS))
    missed = {k: MUTANTS[k] for k, (rc, _) in res.items() if rc == 0}
    assert not missed, "mutants no pin caught: %s" % missed


def test_unmutated_oracle_passes_the_pins():
    env = dict(os.environ)
    env.pop("FOS_ORACLE_MUTANT", None)
    r = subprocess.run([sys.executable, "-m", "pytest", PINS, "-q", "-p", "no:cacheprovider", "-m", "not gpu"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]

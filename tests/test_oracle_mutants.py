"""The oracle's pins must catch plausible mistakes (CPU only).

``oracle.c`` carries planted mistakes behind ``ORACLE_MUTANT=n`` (none in the
default build).  Each mutant is compiled to a scratch library and the pin
suites are re-run against it in a child process; every mutant must make at
least one pin fail.
"""
import concurrent.futures
import os
import subprocess
import sys


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")
PINS = ["tests/test_oracle_codecs.py", "tests/test_oracle_quant.py", "tests/test_oracle_linear.py",
        "tests/test_oracle_weight_only.py", "tests/test_oracle_division.py"]

MUTANTS = {
    1: "f32->bf16 truncates instead of rounding",
    2: "E4M3 ties rounded away from zero",
    3: "E4M3 subnormals flushed to zero",
    4: "int8 quotient truncated instead of rounded",
    5: "W8A8 weight scale not rounded to bf16",
    6: "int8 activation scale absmax/128",
    7: "per-token absmax where a per-group one is due",
    8: "activation byte read as unsigned",
    9: "row epilogue drops the weight scale",
    10: "block weight-scale index transposed",
    11: "block weight scale from one element, not the block max",
    12: "E4M3 row product drops the last input channel",
    13: "weight-only product drops the weight scale",
    14: "weight-only block weight-scale index transposed",
    15: "weight-only product drops the first input channel",
    16: "quotient x * (1 / s) instead of the division x / s",
    17: "activation scale absmax * (1 / qmax) instead of absmax / qmax",
    18: "E4M3 weight scale absmax * (1 / 448) instead of absmax / 448",
}


def _build(n: int, d: str) -> str:
    out = os.path.join(d, f"liboracle_m{n}.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                    f"-DORACLE_MUTANT={n}", SRC, "-o", out, "-lm"], check=True)
    return out


def _run_pins(lib: str) -> int:
    env = dict(os.environ, QL_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu", *PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode


def test_every_planted_mistake_fails_a_pin(tmp_path):
    libs = {n: _build(n, str(tmp_path)) for n in [0, *MUTANTS]}
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
        codes = dict(zip(libs, ex.map(_run_pins, libs.values())))
    assert codes.pop(0) == 0, "the unmutated oracle must pass its pins in the same harness"
    survivors = {n: MUTANTS[n] for n, rc in codes.items() if rc == 0}
    assert not survivors, f"mutants not caught by any pin: {survivors}"

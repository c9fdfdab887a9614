"""The oracle's pins catch plausible mistakes: each mutation in
``tests/oracle_mutations.py`` (a dropped bf16 rounding, ties sent the wrong
way, a wrong E4M3 bias, a bf16 with one bit too many, scales on transposed
blocks, swapped nibbles, a wrong E2M1 table entry, swapped SiLU operands, a
wrong tensor- or activation-scale convention, a dropped tensor scale, a
reversed activation operand; for the LoRA adapters an unrounded rank-r
product, a gate delta added after the activation, a mirrored adapter) is planted in a child pytest process that runs
the oracle's pin tests, and that run must fail.  CPU only."""
import os
import subprocess
import sys

import pytest

from oracle_mutations import MUTATIONS

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
PINS = ["tests/test_oracle_codecs.py", "tests/test_oracle_quant.py", "tests/test_oracle_ffn.py",
        "tests/test_oracle_lora.py"]


def _run(mutation):
    env = dict(os.environ)
    env.pop("FFN_ORACLE_MUTATION", None)
    if mutation:
        env["FFN_ORACLE_MUTATION"] = mutation
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_pins_pass_unmutated():
    r = _run(None)
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(mutation):
    r = _run(mutation)
    assert r.returncode == 1 and ("failed" in r.stdout or "error" in r.stdout), (
        f"pins did not catch {mutation}:\n{r.stdout[-2000:]}")

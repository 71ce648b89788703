"""The pins in test_oracle_pins.py are not vacuous: each of these plausible
mistakes, planted in a copy of the oracle's C source (on the CPU, in a
temporary directory; the oracle itself is untouched), makes at least one pin
fail.  Each mutant is compiled with the oracle's own flags and the pins run
against it in a child process (MOE_ORACLE_LIB)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "bias sign": ("* s + b;", "* s - b;"),
    "bias term dropped in the grouped form": ("+ oracle_bf16_to_f64(bias[r * gpr + g]) * sv;", ";"),
    "adjacent codes swapped on read": ("int64_t o = (int64_t)bits * j;", "int64_t o = (int64_t)bits * (j ^ 1);"),
    "3-bit codes straddling two words cut short": ("if (o % 32 + bits > 32)\n        pair |=",
                                                   "if (0)\n        pair |="),
    "ties to the higher index": ("if (best < 0 || l[e] > l[best])", "if (best < 0 || l[e] >= l[best])"),
    "silu sign": ("return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    "gate and up swapped": ("a[i] = silu(g[i]) * u[i];", "a[i] = silu(u[i]) * g[i];"),
    "weights not renormalised": ("w[i] = p[idx[i]] / s;", "w[i] = p[idx[i]];"),
    "shared-expert gate ignored": ("o[j] += gam * y[j];", "o[j] += y[j];"),
    "residual dropped": ("o[j] = oracle_bf16_to_f64(residual[(int64_t)t * H + j]);", "o[j] = 0.0;"),
    "wrong scale group": ("scale[r * gpr + j / group]", "scale[r * gpr + (j / group + 1) % gpr]"),
    "down uses the up matrix": ("rc = oracle_qmatvec(bits, group, H, I, ex->down.codes",
                                "rc = oracle_qmatvec(bits, group, H, I, ex->up.codes"),
    "rmsnorm without eps": ("sqrt(ss / (double)H + eps)", "sqrt(ss / (double)H)"),
    "bf16 rounding truncates": ("double n = nearbyint(ldexp(a, -qe));", "double n = floor(ldexp(a, -qe));"),
}


def _pins_against(source, tmp_path):
    """Compile `source` as the oracle and run the pins on it; returns the
    child's exit status and output."""
    mutated = tmp_path / "moe_oracle.c"
    mutated.write_text(source)
    lib = tmp_path / "liboracle_variant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC",
                    "-I", os.path.join(ROOT, "oracle"), str(mutated), "-o", str(lib), "-lm"],
                   check=True, capture_output=True)
    env = dict(os.environ, MOE_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        "-x", "-q", "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True)
    return r.returncode, r.stdout


def test_unmodified_copy_passes(tmp_path):
    """Control: the same harness on an unmodified copy passes every pin."""
    rc, out = _pins_against(open(SRC).read(), tmp_path)
    assert rc == 0, out[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) >= 1, f"mutation site not found: {before}"
    rc, out = _pins_against(src.replace(before, after, 1), tmp_path)
    assert rc != 0, f"pins did not catch: {name}\n{out[-2000:]}"

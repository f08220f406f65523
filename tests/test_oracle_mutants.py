"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a temporary copy of oracle/oracle.c (on the
CPU; the repository's oracle is untouched), builds it, and runs the pin suite
against it in a subprocess: the suite must FAIL for every mutant.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "weight block index n%128 instead of n/128":
        ("n / ORC_BLOCK) * KB, K, lut);", "n % ORC_BLOCK) * KB, K, lut);"),
    "last K-block dropped":
        ("for (long kb = 0; kb < KB; ++kb) {", "for (long kb = 0; kb + 1 < KB; ++kb) {"),
    "activation scales read row-major":
        ("sa[kb * sa_stride]", "sa[kb]"),
    "subnormal exponent off by one":
        ("v = ldexp((double)mantissa / 8.0, 1 - 7);", "v = ldexp((double)mantissa / 8.0, 0 - 7);"),
    "sign bit ignored":
        ("lut[code] = sign ? -v : v;", "lut[code] = v;"),
    "K index of B shifted":
        ("p += lut[ak[i]] * lut[bk[i]];", "p += lut[ak[i]] * lut[bk[(i + 1) % ORC_BLOCK]];"),
    "weight scale ignored":
        ("((double)sa[kb * sa_stride] * (double)sb[kb]) * p", "((double)sa[kb * sa_stride]) * p"),
    "k-grouped: every group starts at K-block 0":
        ("        off += Kg;\n", "        off += 0;\n"),
    "k-grouped: group's activation scales taken from K-block 0":
        ("sfa + kb0 * ld_sfa + m", "sfa + m"),
    "bf16: mantissa shifted by one bit":
        ("v.u = (uint32_t)bits << 16;", "v.u = (uint32_t)bits << 15;"),
    "bf16: contiguous rows use group 0's weights":
        ("                bg = m_indices[m];\n", "                bg = 0;\n"),
    "quantiser: scale amax / 240 (the E4M3 'fnuz' maximum)":
        ("float s = amax / 448.0f;", "float s = amax / 240.0f;"),
    "quantiser: encoder rounds ties away from zero":
        ("if (frac > 0.5 || (frac == 0.5 && fmod(lo, 2.0) != 0.0)) r = lo + 1.0;",
         "if (frac >= 0.5) r = lo + 1.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    assert src.count(old) >= 1, "mutation site not found"
    mutated = tmp_path / "oracle_mutant.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "oracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           "-o", str(so), str(mutated), "-lm"])
    env = dict(os.environ, ORACLE_SO=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py"),
                        os.path.join(ROOT, "tests", "test_oracle_quant.py"),
                        os.path.join(ROOT, "tests", "test_oracle_bf16.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch: {name}\n{r.stdout[-2000:]}"

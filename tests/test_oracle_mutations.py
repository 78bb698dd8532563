"""The pins must catch a plausible mistake anywhere in the oracle.

Each case plants one mistake in a temporary copy of oracle/dsa_oracle.c,
builds it, and runs tests/test_oracle_pins.py against that build in a
subprocess (ORACLE_LIB_PATH); the pins must fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dsa_oracle.c")

MUTATIONS = {
    "relu dropped": ("(dot > 0.0 ? dot : 0.0)", "dot"),
    "gqa group h % Hkv": ("int g = h / G;\n        const uint16_t* q = c->Q + (t * c->Hq + h)",
                          "int g = h % c->Hkv;\n        const uint16_t* q = c->Q + (t * c->Hq + h)"),
    "ties to the higher index": ("return (a->s > b->s) - (a->s < b->s);",
                                 "return (a->s < b->s) - (a->s > b->s);"),
    "softmax scale dropped": ("x[i] = scale * dot;", "x[i] = dot;"),
    "weights of the wrong row": ("c->w + t * c->H, c->kI", "c->w, c->kI"),
    "causal bound off by one": ("int64_t n = t + 1;", "int64_t n = t;"),
    "ascending output dropped": ("qsort(out, (size_t)m, sizeof(int32_t), i32_cmp);", ""),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_the_pins(name, tmp_path):
    old, new = MUTATIONS[name]
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation site not found: {name}"
    src = tmp_path / "dsa_oracle.c"
    src.write_text(text.replace(old, new, 1))
    lib = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o",
                           str(lib), str(src), "-lm"])
    env = dict(os.environ, ORACLE_LIB_PATH=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"the pins did not catch: {name}\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout

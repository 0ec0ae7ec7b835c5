"""The pins bind the oracle: each plausible mistake, planted in a copy of the
oracle's C source (never in the oracle itself), makes at least one pin of
tests/test_oracle_pins.py fail.  CPU only."""
import os
import shutil
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dsa_oracle.c")

# (mistake, text of the oracle source, the mistaken text)
MUTATIONS = [
    ("ReLU dropped from the indexer",
     "I += wt[j] * (dot > 0.0 ? dot : 0.0);", "I += wt[j] * dot;"),
    ("ties to the higher position",
     "return (x->s > y->s) - (x->s < y->s);", "return (x->s < y->s) - (x->s > y->s);"),
    ("rope values left out of q . c",
     "for (int x = 0; x < ORACLE_DK; ++x) dot += qv[x] * load_elem(kv, row * ORACLE_DK + x, kv_dtype);",
     "for (int x = 0; x < ORACLE_DV; ++x) dot += qv[x] * load_elem(kv, row * ORACLE_DK + x, kv_dtype);"),
    ("key scale ignored",
     "double ks = idx_dtype == ORACLE_FP8 ? (double)k_scale[row] : 1.0;", "double ks = 1.0;"),
    ("query scale ignored",
     "double qs = idx_dtype == ORACLE_FP8 ? (double)q_scale[(int64_t)t * H_I + j] : 1.0;", "double qs = 1.0;"),
    ("head weights shifted by one head",
     "wt[j] = load_elem(w, (int64_t)t * H_I + j, wdt);", "wt[j] = load_elem(w, (int64_t)t * H_I + (j + 1) % H_I, wdt);"),
    ("e4m3 sign flipped",
     "return sign ? -v : v;", "return sign ? v : -v;"),
    ("softmax scale dropped",
     "z[i] = scale * dot;", "z[i] = dot;"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_a_planted_mistake(tmp_path, name, old, new):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not found once in the oracle source"
    mutant = tmp_path / "dsa_oracle_mutant.c"
    mutant.write_text(src.replace(old, new))
    so = tmp_path / "libdsa_oracle_mutant.so"
    subprocess.check_call(["gcc"] + oracle.GCC_FLAGS + [str(mutant), "-o", str(so), "-lm"])
    env = dict(os.environ, DSA_ORACLE_LIB=str(so), DSA_ORACLE_MUTANT_RUN="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                        os.path.join("tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 1 and " failed" in r.stdout, (
        f"planted mistake '{name}' was not caught by any pin:\n{r.stdout[-3000:]}{r.stderr[-2000:]}")


def test_unmodified_copy_passes_the_pins(tmp_path):
    # the control: the same build and run with the source as it is
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    so = tmp_path / "libdsa_oracle_copy.so"
    subprocess.check_call(["gcc"] + oracle.GCC_FLAGS + [SRC, "-o", str(so), "-lm"])
    env = dict(os.environ, DSA_ORACLE_LIB=str(so), DSA_ORACLE_MUTANT_RUN="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                        os.path.join("tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]

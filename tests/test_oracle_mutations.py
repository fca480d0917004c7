"""The oracle's pins catch plausible mistakes: each mutant below plants one
mistake in a copy of the oracle (a dropped term, a wrong bias, a wrong index,
a missing normalisation, a wrong rounding rule), and the pins of
tests/test_oracle_pins.py (and, for the Python parts, tests/
test_cache_oracle_pins.py) run against it in a child process, which must
fail; the unmutated copy, run the same way, must pass.  Nothing under
oracle/ is modified: a mutant of mla_oracle.c is compiled on its own and
loaded through MLA_ORACLE_LIB; a mutant of a Python part runs in a scratch
copy of the files the pins need.

A mutant's anchor text must occur exactly once in the oracle source: when
the oracle is edited, this test names the anchor to update."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "mla_oracle.c")

MUTANTS = {
    "RoPE term loses its last dimension": (
        "for (int i = ORC_DC; i < ORC_DROW; ++i) acc +=", "for (int i = ORC_DC; i < ORC_DROW - 1; ++i) acc +="),
    "softmax scale left out": ("s[t - t0] = scale * acc;", "s[t - t0] = acc;"),
    "lse without the row max": ("*lse = m + log(l);", "*lse = log(l);"),
    "E4M3 subnormal exponent off by one": ("ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)"),
    "E4M3 normal bias off by one": ("ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)"),
    "merge weights relative to the max, not the merged lse": ("double w = exp(li - L);", "double w = exp(li - M);"),
    "values read from the first block only": (
        "int32_t blk = table_row[t / ORC_BLOCK];", "int32_t blk = table_row[0];"),
    "last output column not normalised": (
        "for (int i = 0; i < ORC_DC; ++i) o[i] /= l;", "for (int i = 0; i < ORC_DC - 1; ++i) o[i] /= l;"),
    "query absorption uses the next head's W_UK": (
        "const uint16_t *w = w_uk + ((int64_t)h * 128 + d) * ORC_DC;",
        "const uint16_t *w = w_uk + ((int64_t)((h + 1) % H) * 128 + d) * ORC_DC;"),
    "output absorption drops the last latent column": (
        "for (int c = 0; c < ORC_DC; ++c) acc += orc_bf16_to_f64(w[c]) * orc_bf16_to_f64(o[c]);",
        "for (int c = 0; c < ORC_DC - 1; ++c) acc += orc_bf16_to_f64(w[c]) * orc_bf16_to_f64(o[c]);"),
}


# mistakes planted in the oracle's Python parts (file under oracle/, anchor, replacement)
PY_MUTANTS = {
    "RoPE rotation with a wrong sign": (
        "naive.py", "out[..., 1::2] = x0 * s + x1 * c", "out[..., 1::2] = x0 * s - x1 * c"),
    "unabsorbed values formed with W_UK": (
        "naive.py", "v = c_kv @ w_uv[h].T", "v = c_kv @ w_uk[h].T"),
    "E4M3 ties rounded to the odd code": (
        "cache.py", "score = np.where(cand, 1 + 2 * even[None, :] + same_sign, 0)",
        "score = np.where(cand, 1 + 2 * (1 - even[None, :]) + same_sign, 0)"),
    "appended row one slot late": (
        "cache.py", "return blocks, (pos % BLOCK).astype(np.int64), rows",
        "return blocks, ((pos + 1) % BLOCK).astype(np.int64), rows"),
}

# the files a child run of the pins needs, copied into a scratch tree
_TREE = ["oracle/__init__.py", "oracle/naive.py", "oracle/cache.py", "oracle/mla_oracle.c",
         "mla_latent_kv_25_b200/__init__.py", "mla_latent_kv_25_b200/inputs.py",
         "mla_latent_kv_25_b200/layout.py", "tests/__init__.py", "tests/conftest.py", "tests/_util.py",
         "tests/test_oracle_pins.py", "tests/test_cache_oracle_pins.py"]


def _tree_with(where, rel, old, new):
    import shutil
    for f in _TREE + [os.path.join("tests", "golden", g) for g in os.listdir(os.path.join(ROOT, "tests", "golden"))]:
        src = os.path.join(ROOT, f)
        if not os.path.exists(src):
            continue
        dst = where / f
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copyfile(src, dst)
    target = where / "oracle" / rel
    text = target.read_text()
    assert text.count(old) == 1, f"anchor not unique in oracle/{rel}: {old}"
    target.write_text(text.replace(old, new))
    env = dict(os.environ)
    env.pop("MLA_ORACLE_LIB", None)
    return subprocess.run([sys.executable, "-m", "pytest", str(where / "tests" / "test_oracle_pins.py"),
                           str(where / "tests" / "test_cache_oracle_pins.py"), "-x", "-q",
                           "-p", "no:cacheprovider"], cwd=str(where), env=env,
                          capture_output=True, text=True, timeout=900)


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_pins_catch_the_python_mutant(name, tmp_path):
    rel, old, new = PY_MUTANTS[name]
    r = _tree_with(tmp_path, rel, old, new)
    assert "passed" in r.stdout or "failed" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
    assert r.returncode != 0, f"mutant '{name}' passed every pin"


def test_scratch_tree_without_a_mutant_passes_the_pins(tmp_path):
    r = _tree_with(tmp_path, "naive.py", "import numpy as np", "import numpy as np")
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


def _build(src_text, where):
    c = where / "oracle_copy.c"
    so = where / "liboracle_copy.so"
    c.write_text(src_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
                    "-o", str(so), str(c), "-lm"], check=True, capture_output=True, text=True, timeout=120)
    return so


def _pins(lib):
    env = dict(os.environ, MLA_ORACLE_LIB=str(lib))
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                           "-x", "-q", "-p", "no:cacheprovider"], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_unmutated_copy_passes_the_pins(tmp_path):
    r = _pins(_build(open(SRC).read(), tmp_path))
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_the_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"anchor of mutant '{name}' not unique in the oracle: {old}"
    r = _pins(_build(src.replace(old, new), tmp_path))
    assert r.returncode != 0, f"mutant '{name}' passed every pin"

"""The pins catch plausible mistakes in the oracle (CPU only).

Each case plants one mistake in a temporary copy of ``oracle/gdn2_oracle.c``
(a dropped gate, a wrong sign, a transposed or swapped operand, a wrong step
order, a skipped token) and runs the pin tests against the mutated copy; at
least one pin must fail.  The repository's oracle is never modified.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gdn2_oracle.c")

FWD = [
    # step 1: no decay
    ("for (int64_t i = 0; i < dk; ++i) a[i] = exp(scalar_decay ? gt[0] : gt[i]);",
     "for (int64_t i = 0; i < dk; ++i) a[i] = 1.0;"),
    # step 3: erase without the gate b
    ("            for (int64_t i = 0; i < dk; ++i) x[i] = (scalar_gates ? bt[0] : bt[i]) * kt[i];\n"
     "            for (int64_t i = 0; i < dk; ++i)\n"
     "                for (int64_t j = 0; j < dv; ++j) S[i * dv + j] -= x[i] * r[j];",
     "            for (int64_t i = 0; i < dk; ++i) x[i] = kt[i];\n"
     "            for (int64_t i = 0; i < dk; ++i)\n"
     "                for (int64_t j = 0; j < dv; ++j) S[i * dv + j] -= x[i] * r[j];"),
    # step 3: wrong sign of the erase
    ("for (int64_t j = 0; j < dv; ++j) S[i * dv + j] -= x[i] * r[j];",
     "for (int64_t j = 0; j < dv; ++j) S[i * dv + j] += x[i] * r[j];"),
    # step 4: the write uses the erase gate
    ("for (int64_t i = 0; i < dk; ++i) p[i] = (scalar_gates ? wt[0] : wt[i]) * kt[i];",
     "for (int64_t i = 0; i < dk; ++i) p[i] = (scalar_gates ? bt[0] : bt[i]) * kt[i];"),
    # step 2: erase read with the query instead of the key
    ("for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * kt[i];",
     "for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * qt[i];"),
    # step 5: read with the key
    ("for (int64_t j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * qt[i];",
     "for (int64_t j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * kt[i];"),
    # gist.science form: erase read with k instead of b.k
    ("for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * x[i];",
     "for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * kt[i];"),
    # gist.science form: erase sides swapped (read with k, erase along b.k)
    ("                for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * x[i];\n"
     "            for (int64_t i = 0; i < dk; ++i)\n"
     "                for (int64_t j = 0; j < dv; ++j) S[i * dv + j] -= kt[i] * r[j];",
     "                for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * kt[i];\n"
     "            for (int64_t i = 0; i < dk; ++i)\n"
     "                for (int64_t j = 0; j < dv; ++j) S[i * dv + j] -= x[i] * r[j];"),
    # gist.science form: write gate on the key axis, (w.k) v^T instead of k (w.v)^T
    ("            for (int64_t j = 0; j < dv; ++j) p[j] = (scalar_gates ? wt[0] : wt[j]) * vt[j];\n"
     "            for (int64_t i = 0; i < dk; ++i)\n"
     "                for (int64_t j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * p[j];",
     "            for (int64_t i = 0; i < dk; ++i)\n"
     "                for (int64_t j = 0; j < dv; ++j)\n"
     "                    S[i * dv + j] += (scalar_gates ? wt[0] : wt[i]) * kt[i] * vt[j];"),
]
BWD = [
    ("const double gb = G[i * dv + j] + y[i] * dr[j];", "const double gb = G[i * dv + j];"),
    ("ag += gb * sbar;", "ag += gb * S_prev[i * dv + j];"),
    ("dvt[j] = wj * dz[j];", "dvt[j] = dz[j];"),
    ("dkt[i] = dy[i] + bi * dx[i] + wi * dp[i];", "dkt[i] = dy[i] + bi * dx[i] + dp[i];"),
    ("for (int64_t t = t1 - 1; t >= t0; --t) {", "for (int64_t t = t1 - 1; t > t0; --t) {"),
    ("ax -= G[i * dv + j] * r[j];", "ax += G[i * dv + j] * r[j];"),
]


def _run_pins(tmp, src_text, pin_file):
    d = os.path.join(tmp, "m")
    if os.path.exists(d):
        shutil.rmtree(d)
    os.makedirs(os.path.join(d, "tests"))
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "*.so.tmp*", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(d, "tests", "golden"))
    for f in ("conftest.py", pin_file):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(d, "tests", f))
    with open(os.path.join(d, "oracle", "gdn2_oracle.c"), "w") as f:
        f.write(src_text)
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join("tests", pin_file)], cwd=d, capture_output=True, text=True, env=env,
                       timeout=600)
    return r.returncode, r.stdout[-400:]


@pytest.mark.parametrize("k", range(len(FWD)))
def test_forward_pins_catch_planted_mistake(tmp_path, k):
    src = open(SRC).read()
    a, b = FWD[k]
    assert src.count(a) == 1, a
    rc, out = _run_pins(str(tmp_path), src.replace(a, b), "test_oracle_pins.py")
    assert rc != 0, f"pins passed with a planted mistake:\n{b}\n{out}"


@pytest.mark.parametrize("k", range(len(BWD)))
def test_backward_pins_catch_planted_mistake(tmp_path, k):
    src = open(SRC).read()
    a, b = BWD[k]
    assert src.count(a) == 1, a
    rc, out = _run_pins(str(tmp_path), src.replace(a, b), "test_oracle_bwd_pins.py")
    assert rc != 0, f"pins passed with a planted mistake:\n{b}\n{out}"


@pytest.mark.parametrize("pin_file", ["test_oracle_pins.py", "test_oracle_bwd_pins.py"])
def test_unmutated_copy_passes(tmp_path, pin_file):
    rc, out = _run_pins(str(tmp_path), open(SRC).read(), pin_file)
    assert rc == 0, out

"""The oracle's pins catch plausible slips: each mutation below plants one
mistake in a copy of the oracle's C source (on the CPU), rebuilds it, and runs
the pin suite against the copy, which must fail.

The slips are the kinds of mistake that reading the pages could produce: min
and max swapped, the wrong head-to-group mapping, the log-gate added with the
wrong sign, the softmax scale dropped, the local-block range shifted, the
tie-break reversed, the gate's average over the whole block instead of the
valid tokens, no length mask, the query projection transposed, the gate's
1/sqrt(dg) dropped, the gate softmax over all N blocks instead of the C = N-1
historical ones, and an unnormalised split merge.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

import pytest

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "quest min/max swapped": ("mn[o] = lo;\n                    mx[o] = hi;",
                              "mn[o] = hi;\n                    mx[o] = lo;"),
    "wrong GQA mapping": ("int qh = g * G + hh;", "int qh = hh * c->H_kv + g;"),
    "log-gate sign": ("l[nt] = dot * scale + bj;", "l[nt] = dot * scale - bj;"),
    "softmax scale dropped": ("l[nt] = dot * scale + bj;", "l[nt] = dot + bj;"),
    "local range shifted": ("for (int j = N - L; j < N; ++j)\n                chosen[cnt++] = j;",
                            "for (int j = N - L + 1; j <= N; ++j)\n                chosen[cnt++] = j;"),
    "tie-break reversed": ("return a->j - b->j;", "return b->j - a->j;"),
    "gate average over the whole block": ("p[2 * d + ch] = sum / (double)(t1 - t0);",
                                          "p[2 * d + ch] = sum / (double)c->b;"),
    "no length mask": ("t < (j + 1) * c->b && t < len; ++t) {", "t < (j + 1) * c->b; ++t) {"),
    "query projection transposed": ("acc += (double)Wq[(int64_t)r * d + ch] *",
                                    "acc += (double)Wq[(int64_t)ch * dg + r] *"),
    "gate 1/sqrt(dg) dropped": ("u[j] = acc / sqrt((double)dg);", "u[j] = acc;"),
    "gate softmax over N blocks": ("int C = N - 1; /* number of historical blocks */", "int C = N;"),
    "unnormalised merge": ("double w = exp(lse_part[r * S + sp] - m) / z;",
                           "double w = exp(lse_part[r * S + sp] - m);"),
}


def _run_pins_on_copy(tmp_path, old=None, new=None):
    """Copy the oracle and the tests, plant `old` -> `new` in the C source, run the pins."""
    shutil.copytree(os.path.join(REPO, "oracle"), tmp_path / "oracle",
                    ignore=shutil.ignore_patterns("_liboracle.so*", "__pycache__"))
    shutil.copytree(os.path.join(REPO, "tests"), tmp_path / "tests",
                    ignore=shutil.ignore_patterns("__pycache__"))
    if old is not None:
        src = tmp_path / "oracle" / "sba_oracle.c"
        text = src.read_text()
        assert text.count(old) == 1, old
        src.write_text(text.replace(old, new))
    env = dict(os.environ, PYTHONPATH=os.pathsep.join([str(tmp_path), REPO]))
    return subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q",
                           "-p", "no:cacheprovider"], cwd=tmp_path, env=env, capture_output=True, text=True,
                          timeout=600)


def test_pins_pass_on_an_unmodified_copy(tmp_path):
    """Control: the harness itself leaves the pins green."""
    r = _run_pins_on_copy(tmp_path)
    assert r.returncode == 0, (r.stdout + r.stderr)[-400:]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_slip(name, tmp_path):
    r = _run_pins_on_copy(tmp_path, *MUTATIONS[name])
    tail = (r.stdout + r.stderr)[-400:]
    assert r.returncode == 1, f"{name}: the pins did not fail (rc {r.returncode})\n{tail}"
    assert "failed" in r.stdout, tail

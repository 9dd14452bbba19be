"""Planted mistakes in the oracle must fail its pins (CPU only).

Each mutant is a copy of oracle/dbsa_oracle.c with one plausible error
(a sign, an index, a dropped term, a wrong position), compiled on the side;
the pin suite is run against it in a subprocess and must fail.
"""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dbsa_oracle.c")

MUTANTS = {
    "rope_sign": ("y[i] = x[i] * c - x[i + h] * s;", "y[i] = x[i] * c + x[i + h] * s;"),
    "rope_freq": ("double w = pow(theta, -2.0 * (double)i / (double)d);",
                  "double w = pow(theta, -1.0 * (double)i / (double)d);"),
    "window_off_by_one": ("int is_prev = (bs >= bt - j) && (bs < bt);",
                          "int is_prev = (bs > bt - j) && (bs < bt);"),
    "sink_dropped": ("case ORC_PATTERN_SINK_PREV_SELF: return is_sink || is_prev || is_self;",
                     "case ORC_PATTERN_SINK_PREV_SELF: return is_prev || is_self;"),
    "not_causal": ("if (s > t) return 0; /* causal */", "if (s > t + 1) return 0;"),
    "scale": ("if (scale <= 0.0) scale = 1.0 / sqrt((double)d);\n    int32_t g = Hq / Hkv;\n    int32_t bad = 0;",
              "if (scale <= 0.0) scale = 1.0 / (double)d;\n    int32_t g = Hq / Hkv;\n    int32_t bad = 0;"),
    "gqa_mapping": ("        int32_t c = h / g;\n        /* explicit boolean mask row */",
                    "        int32_t c = h % Hkv;\n        /* explicit boolean mask row */"),
    "query_position": ("orc_rope(x, d, (double)(Tg + tu), theta, qr);",
                       "orc_rope(x, d, (double)(Tg + tu + 1), theta, qr);"),
    "fresh_positions": ("map[2 * p + 1] = (int32_t)p;", "map[2 * p + 1] = (int32_t)s;"),
    "tail_position": ("orc_rope(x, d, (double)(Tg + w), theta, kr + p * d);",
                      "orc_rope(x, d, (double)(w), theta, kr + p * d);"),
}


def _run_mutant(name, tmp):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path_c = os.path.join(tmp, name + ".c")
    path_so = os.path.join(tmp, name + ".so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           "-o", path_so, path_c, "-lm"])
    env = dict(os.environ, DBSA_ORACLE_LIB=path_so, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    return name, r.returncode


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(os.sched_getaffinity(0)))) as ex:
            results = list(ex.map(lambda n: _run_mutant(n, tmp), MUTANTS))
    survivors = [n for n, rc in results if rc == 0]
    assert not survivors, "pins did not catch: %s" % survivors

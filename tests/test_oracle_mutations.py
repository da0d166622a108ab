"""The oracle's pins catch plausible mistakes: each test plants one mistake in
a temporary copy of the oracle source, builds that copy, runs the pin suite
against it in a child process, and expects the suite to fail.  A control
run on an unmodified copy must pass, so the failures come from the planted
mistakes and not from the copying.  CPU only; the real oracle is untouched."""
import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "eblc_oracle.c")

# (what the mistake is, text in the source, replacement)
MUTATIONS = [
    ("zigzag sign", "return (uint32_t)(-2 * v - 1);", "return (uint32_t)(-2 * v + 1);"),
    ("no Lorenzo reset at block starts", "int32_t prev = 0; /* Lorenzo", "static int32_t prev = 0; /* Lorenzo"),
    ("width off by one", "++w;", "w += (acc > 1) ? 1 : 2;"),
    ("truncation instead of rounding", "return (int32_t)nearbyintf(y);", "return (int32_t)y;"),
    ("int range limit 2^31", "1073741824.0f", "2147483648.0f"),
    ("strict bound test", "fabs((double)x - (double)xr) <= eb", "fabs((double)x - (double)xr) < eb"),
    ("eb from vmax + vmin", "bound * ((double)vmax - (double)vmin)", "bound * ((double)vmax + (double)vmin)"),
    ("step = eb", "*step_out = (float)two_eb;", "*step_out = (float)eb;"),
    ("reversed pack order", "uint64_t v = (uint64_t)z[j] << sh;", "uint64_t v = (uint64_t)z[cnt - 1 - j] << sh;"),
    ("index outlier count", "outl_before += mc;", "outl_before += 0;"),
    ("record without values", "rec += 2 * mc;", "rec += mc;"),
    ("no canonical +0", "*vmin_out = lo + 0.0f;", "*vmin_out = lo;"),
    ("inverse zigzag", "return (int32_t)(-(int64_t)(z / 2u) - 1);", "return (int32_t)(-(int64_t)(z / 2u));"),
    ("dequantisation", "return (float)q * step; }", "return (float)q * step * 1.0000001f; }"),
    ("given range ignored", "if (!abs_mode && range) {", "if (!abs_mode && range && 0) {"),
    ("Lorenzo stencil corner sign", "acc = ((a + b + c) & 1u) ? acc - v : acc + v;",
     "acc = ((a + b) & 1u) ? acc - v : acc + v;"),
    ("Lorenzo inverse along y", "q[e] = (int32_t)((uint32_t)q[e] + (uint32_t)q[e - be[2]]);",
     "q[e] = (int32_t)((uint32_t)q[e] + (uint32_t)q[e - 1]);"),
    ("block z index", "uint64_t z = cz * ce[0] + iz * be[0] + ez;", "uint64_t z = cz * ce[0] + iz * be[0];"),
    ("bitshuffle plane order", "out[b * G + g] = word;", "out[g * 32 + b] = word;"),
    ("zero-elimination bitmap order", "out[j / 32] |= 1u << (j % 32);", "out[j / 32] |= 1u << (31 - j % 32);"),
    ("chunk Diff without reset", "int32_t prev = 0;  /* Diff: 0 before the chunk's first code */",
     "static int32_t prev = 0;  /* Diff: 0 before the chunk's first code */"),
    ("verbatim when larger", "int raw = r >= mp;", "int raw = r > mp + 1000000;"),
    ("repetition predecessor of word 0", "uint32_t pred = j ? in[j - 1] : 0u;", "uint32_t pred = j ? in[j - 1] : in[0];"),
    ("repetition inverse fills zeros", "        out[j] = last;",
     "        out[j] = ((in[j / 32] >> (j % 32)) & 1u) ? last : 0u;"),
    ("repetition coder flag", "(coder ? ORC_FLAG_RRE : 0u)", "(coder ? 0u : 0u)"),
]


def _run_pins(src_path: str) -> subprocess.CompletedProcess:
    env = dict(os.environ, EBLC_ORACLE_SRC=src_path, PYTHONDONTWRITEBYTECODE="1")
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                           os.path.join(ROOT, "tests", "test_oracle_nd_pins.py"),
                           os.path.join(ROOT, "tests", "test_oracle_chunked_pins.py"),
                           "-x", "-q", "-p", "no:cacheprovider", "-k", "not fuzz"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


def test_planted_mistakes_fail_the_pins(tmp_path):
    original = open(SRC).read()
    jobs = {}
    control = tmp_path / "control.c"
    control.write_text(original)
    jobs["control"] = str(control)
    for k, (what, old, new) in enumerate(MUTATIONS):
        assert original.count(old) == 1, f"mutation anchor for {what!r} not found exactly once"
        path = tmp_path / f"m{k}.c"
        path.write_text(original.replace(old, new, 1))
        jobs[what] = str(path)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = dict(zip(jobs, ex.map(_run_pins, jobs.values())))
    ctl = results.pop("control")
    assert ctl.returncode == 0, "the unmodified copy must pass the pins:\n" + ctl.stdout[-2000:]
    survived = [what for what, r in results.items() if r.returncode == 0]
    assert not survived, f"planted mistakes the pins did not catch: {survived}"
    assert open(SRC).read() == original  # the real oracle is untouched

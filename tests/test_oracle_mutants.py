"""The oracle's pins must catch plausible mistakes in the oracle itself.

Each case plants one mistake in a copy of oracle/attn_oracle.c (a dropped
term, a wrong sign, offset or index, a swapped operand), builds it on the CPU
and runs the pin suites (tests/test_oracle_pins.py, tests/test_oracle_bound.py)
against it in a child process: at least one pin must fail.  The oracle in the
repository is untouched.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "attn_oracle.c")

MUTANTS = [
    # (what, exact text in the oracle, planted replacement)
    ("causal offset dropped", "return j <= i + (Nkv - Nq);", "return j <= i;"),
    ("causal diagonal excluded", "return j <= i + (Nkv - Nq);", "return j < i + (Nkv - Nq);"),
    ("block predicate inverted", "(j / ORA_GRAIN)] != 0;", "(j / ORA_GRAIN)] == 0;"),
    ("scale dropped", "S[j] = scale * acc;", "S[j] = acc;"),
    ("max not subtracted", "exp(S[j] - m);", "exp(S[j]);"),
    ("LSE without the log", "*lse = m + log(l);", "*lse = m + l;"),
    ("modulo GQA mapping", "int hkv = hq / G;", "int hkv = hq % Hkv;"),
    ("V rows reversed", "o[t] += S[j] * ld(v, dtype, kv_off + (size_t)j * kv_row_stride + t);",
     "o[t] += S[j] * ld(v, dtype, kv_off + (size_t)(nkeys - 1 - j) * kv_row_stride + t);"),
    ("decode drops the newest key", "seqlens[b], d, scale, dtype,",
     "(seqlens[b] > 1 ? seqlens[b] - 1 : seqlens[b]), d, scale, dtype,"),
    ("merge weights not normalised", "double w = exp(lse_parts[s] - L);", "double w = exp(lse_parts[s] - m);"),
    ("backward: D term dropped", "double ds = P[j] * (dP[j] - D);", "double ds = P[j] * dP[j];"),
    ("backward: dK without the scale", "dk[kj + t] += scale * ds * ld(q, dtype, q_off + t);",
     "dk[kj + t] += ds * ld(q, dtype, q_off + t);"),
    ("backward: dV from dS", "dv[kj + t] += P[j] * ld(dout, dtype, q_off + t);",
     "dv[kj + t] += ds * ld(dout, dtype, q_off + t);"),
    ("key mean over Nkv + 1", "for (int t = 0; t < d; ++t) m[t] /= Nkv;",
     "for (int t = 0; t < d; ++t) m[t] /= (Nkv + 1);"),
    ("frame rule: next frame instead of previous", "return fj == 0 || fj == fi || fj == fi - 1;",
     "return fj == 0 || fj == fi || fj == fi + 1;"),
    ("frame rule: reference frame dropped", "return fj == 0 || fj == fi || fj == fi - 1;",
     "return fj == fi || fj == fi - 1;"),
    ("radius squared", "radius[(size_t)b * Hkv + h] = sqrt(r2);", "radius[(size_t)b * Hkv + h] = r2;"),
    ("bound rule inverted", "int use_bound = 2.0 * M * 1.4426950408889634 <= limit2;",
     "int use_bound = 2.0 * M * 1.4426950408889634 > limit2;"),
    ("per-row dQ: D term dropped", "double ds = S[j] * (dP[j] - D);", "double ds = S[j] * dP[j];"),
    ("per-row dQ: K row misindexed",
     "for (int t = 0; t < d; ++t) out[t] += scale * ds * ld(k, dtype, kv_base + (size_t)j * kv_stride + t);",
     "for (int t = 0; t < d; ++t) out[t] += scale * ds * ld(k, dtype, kv_base + (size_t)(Nkv - 1 - j) * kv_stride + t);"),
]

RUNNER = """
import sys
sys.path.insert(0, {root!r})
import oracle
oracle._SRC, oracle._LIB_PATH = {src!r}, {lib!r}
import pytest
sys.exit(pytest.main(["-x", "-q", "-p", "no:cacheprovider", "--rootdir", {root!r},
                      {pins!r}, {bound!r}]))
"""


def _run_mutant(what, old, new, src, workdir):
    """Build one mutant and run the pins against it; returns (what, exit code, output tail)."""
    assert old in src, f"mutation site not found: {old}"
    os.makedirs(workdir, exist_ok=True)
    msrc, mlib = os.path.join(workdir, "attn_oracle.c"), os.path.join(workdir, "liboracle.so")
    with open(msrc, "w") as f:
        f.write(src.replace(old, new))
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", mlib, msrc, "-lm"], check=True)
    code = RUNNER.format(root=ROOT, src=msrc, lib=mlib, pins=os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                         bound=os.path.join(ROOT, "tests", "test_oracle_bound.py"))
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=900, cwd=ROOT, env=env)
    return what, r.returncode, r.stdout[-1500:]


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_pins_catch_every_planted_mistake(tmp_path):
    """Every mutant makes at least one pin fail (pytest exit code 1); the
    mutants run four at a time."""
    from concurrent.futures import ThreadPoolExecutor
    with open(SRC) as f:
        src = f.read()
    with ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(lambda im: _run_mutant(*im[1], src, str(tmp_path / f"m{im[0]}")), enumerate(MUTANTS)))
    survivors = [(what, rc, out) for what, rc, out in results if rc != 1]
    assert not survivors, "\n".join(f"{w}: exit {rc}\n{out}" for w, rc, out in survivors)

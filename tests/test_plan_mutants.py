"""The host planner's checks must catch plausible mistakes in the planner.

Each case plants one mistake in a copy of exact_io_aware_sm_b200/csrc/plan.cpp
and builds it with g++ alone (through tests/plan_shim.cpp, a test-only C entry
point with attn_plan's output format).  Three checks then run against the
mutant: the oracle's schedule checker on plans of every mask kind (rows
partitioned, KV tiles disjoint, exactly the allowed keys covered, no
predicate-free tile holding a masked element), tests/plan_pairs_check.cpp (the
pair invariants the kernel relies on) and tests/plan_recut_check.cpp (the
two-segment re-cut covers exactly the planned keys).  At least one must fail;
the unmodified planner must pass all three.
"""
import ctypes
import os
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_io_aware_sm_b200", "csrc")
TESTS = os.path.join(ROOT, "tests")

MUTANTS = [
    ("causal: last tile of a row dropped", "if (c0 > last_row + off) break;", "if (c0 >= last_row + off) break;"),
    ("causal: diagonal tile marked full", "full = (c0 + nreal - 1) <= r0 + off;",
     "full = (c0 + nreal - 1) <= r0 + off + 16;"),
    ("tile past Nkv without a predicate", "const bool partial = !full || nc != nreal;", "const bool partial = !full;"),
    ("block: rows merged whatever their map rows",
     "while (br1 < nbr && std::memcmp(rowp, block_map + static_cast<size_t>(br1) * nbc, nbc) == 0)",
     "while (br1 < nbr)"),
    ("block: tile past Nkv without a predicate", "const bool partial = c0 + nc > Nkv;", "const bool partial = false;"),
    ("re-cut: head of the next span counted twice", "      off = n1;\n", "      off = 0;\n"),
    ("pairs: slot flags swapped", "if (a && k < a->n_kv && plan.kv[a->first_kv + k].partial) flags |= 1;",
     "if (a && k < a->n_kv && plan.kv[a->first_kv + k].partial) flags |= 2;"),
    ("pairs: nesting accepts a longer slot A", "    if (a.n_kv > b.n_kv) return false;\n", "\n"),
    ("pairs: shortest first", "return out->pairs[x].nB > out->pairs[y].nB;",
     "return out->pairs[x].nB < out->pairs[y].nB;"),
]


def _cases():
    rng = np.random.default_rng(4242)
    out = [(oracle.MASK_CAUSAL, None, n, m) for n, m in [(1024, 1024), (333, 200), (200, 333), (17, 5), (1, 1),
                                                         (300, 300), (130, 1000)]]
    out += [(oracle.MASK_NONE, None, n, m) for n, m in [(250, 77), (256, 256), (129, 300)]]
    for _ in range(12):
        Nq, Nkv = (int(x) for x in rng.integers(1, 600, size=2))
        bm = (rng.random(((Nq + 15) // 16, (Nkv + 15) // 16)) < rng.uniform(0.1, 0.9)).astype(np.uint8)
        if rng.random() < 0.5:
            for r in range(1, bm.shape[0]):
                if rng.random() < 0.7:
                    bm[r] = bm[r - 1]
        out.append((oracle.MASK_BLOCK, bm, Nq, Nkv))
    out.append((oracle.MASK_BLOCK, oracle.frame_block_map(6, 80), 480, 480))
    out.append((oracle.MASK_BLOCK, oracle.frame_block_map(4, 1040), 4160, 4160))
    return out


def _build(plan_src, workdir):
    os.makedirs(workdir, exist_ok=True)
    shutil.copy(os.path.join(CSRC, "plan.h"), workdir)
    with open(os.path.join(workdir, "plan.cpp"), "w") as f:
        f.write(plan_src)
    cc = ["g++", "-O2", "-std=c++17", "-I", workdir]
    lib = os.path.join(workdir, "libplan.so")
    subprocess.run(cc + ["-shared", "-fPIC", "-Wl,-Bsymbolic", "-o", lib, os.path.join(TESTS, "plan_shim.cpp"),
                         os.path.join(workdir, "plan.cpp")], check=True)
    exes = []
    for check in ("plan_pairs_check.cpp", "plan_recut_check.cpp"):
        exe = os.path.join(workdir, check[:-4])
        subprocess.run(cc + ["-o", exe, os.path.join(TESTS, check), os.path.join(workdir, "plan.cpp")], check=True)
        exes.append(exe)
    return lib, exes


def _schedule_failures(lib_path, cases):
    L = ctypes.CDLL(lib_path)
    P, I = ctypes.c_void_p, ctypes.c_int
    L.shim_plan.argtypes = [I, P, I, I, P, I, P, I, P, P]
    bad = 0
    for kind, bm, Nq, Nkv in cases:
        bmc = None if bm is None else np.ascontiguousarray(bm, np.uint8)
        bmp = None if bmc is None else bmc.ctypes.data_as(P)
        nq, nk = ctypes.c_int(0), ctypes.c_int(0)
        L.shim_plan(kind, bmp, Nq, Nkv, None, 0, None, 0, ctypes.byref(nq), ctypes.byref(nk))
        qt = np.zeros((max(nq.value, 1), 4), np.int32)
        kt = np.zeros((max(nk.value, 1), 3), np.int32)
        L.shim_plan(kind, bmp, Nq, Nkv, qt.ctypes.data_as(P), nq.value, kt.ctypes.data_as(P), nk.value,
                    ctypes.byref(nq), ctypes.byref(nk))
        if oracle.check_schedule(kind, bm, Nq, Nkv, qt[:nq.value], kt[:nk.value]) != 0:
            bad += 1
    return bad


def _run(plan_src, workdir, cases):
    lib, exes = _build(plan_src, workdir)
    sched = _schedule_failures(lib, cases)
    rc = [subprocess.run([e], capture_output=True, text=True, timeout=300).returncode for e in exes]
    return sched, rc


pytestmark = pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")


def test_unmodified_planner_passes_every_check(tmp_path):
    with open(os.path.join(CSRC, "plan.cpp")) as f:
        src = f.read()
    sched, rc = _run(src, str(tmp_path / "orig"), _cases())
    assert sched == 0 and rc == [0, 0], (sched, rc)


def test_checks_catch_every_planted_mistake(tmp_path):
    with open(os.path.join(CSRC, "plan.cpp")) as f:
        src = f.read()
    for what, old, new in MUTANTS:
        assert src.count(old) == 1, f"mutation site not unique or missing: {what}"
    cases = _cases()

    def one(im):
        i, (what, old, new) = im
        sched, rc = _run(src.replace(old, new), str(tmp_path / f"m{i}"), cases)
        return what, sched, rc

    with ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(one, enumerate(MUTANTS)))
    survivors = [(w, s, rc) for w, s, rc in results if s == 0 and rc == [0, 0]]
    assert not survivors, f"mutants no check caught: {survivors}"

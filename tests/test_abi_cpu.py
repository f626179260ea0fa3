"""Host-side checks of the C-ABI library (no GPU needed).

* libattn_b200.so loads and exports every function declared in include/attn.h;
* block maps, tile classes and tile schedules are bit-exact with the oracle's
  brute-force element enumeration;
* argument errors come back as status codes before any device work.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import exact_io_aware_sm_b200 as eio
import oracle
from exact_io_aware_sm_b200 import build as ebuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_lib():
    ebuild.build()
    return eio.lib()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(attn_[a-z0-9_]+)\s*\(",
                                text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert "attn_fwd" in names and "attn_decode" in names and len(names) >= 8
    L = ctypes.CDLL(eio.LIB_PATH)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert eio.version().startswith("exact_io_aware_sm_b200")


def test_frame_block_map_bit_exact():
    for F, L in [(24, 1040), (3, 16), (5, 48), (2, 1040), (7, 112)]:
        assert np.array_equal(eio.frame_block_map(F, L), oracle.frame_block_map(F, L))
    with pytest.raises(eio.AttnError) as ei:
        eio.frame_block_map(4, 1000)  # not a multiple of 16
    assert ei.value.code == 2


def _random_map(rng, nbr, nbc, p):
    return (rng.random((nbr, nbc)) < p).astype(np.uint8)


CLASSIFY_CASES = [
    (oracle.MASK_NONE, None, 300, 200, 128, 128),
    (oracle.MASK_CAUSAL, None, 1024, 1024, 128, 128),
    (oracle.MASK_CAUSAL, None, 1000, 1300, 128, 64),
    (oracle.MASK_CAUSAL, None, 1300, 1000, 100, 37),
    (oracle.MASK_CAUSAL, None, 17, 5, 16, 16),
]


@pytest.mark.parametrize("case", CLASSIFY_CASES)
def test_classify_matches_oracle(case):
    kind, bm, Nq, Nkv, tq, tk = case
    assert np.array_equal(eio.classify(kind, bm, Nq, Nkv, tq, tk),
                          oracle.classify(kind, bm, Nq, Nkv, tq, tk))


@pytest.mark.parametrize("seed", range(4))
def test_classify_block_maps_match_oracle(seed):
    rng = np.random.default_rng(seed)
    Nq, Nkv = int(rng.integers(1, 700)), int(rng.integers(1, 700))
    bm = _random_map(rng, (Nq + 15) // 16, (Nkv + 15) // 16, rng.uniform(0.1, 0.9))
    for tq, tk in [(128, 128), (16, 16), (64, 32), (48, 80), (7, 129)]:
        assert np.array_equal(eio.classify(oracle.MASK_BLOCK, bm, Nq, Nkv, tq, tk),
                              oracle.classify(oracle.MASK_BLOCK, bm, Nq, Nkv, tq, tk))


def test_classify_frame_config():
    bm = eio.frame_block_map(24, 1040)
    for t in (128, 16):
        assert np.array_equal(eio.classify(oracle.MASK_BLOCK, bm, 24960, 24960, t, t),
                              oracle.classify(oracle.MASK_BLOCK, bm, 24960, 24960, t, t))


PLAN_CASES = [
    (oracle.MASK_NONE, 256, 256),
    (oracle.MASK_NONE, 250, 77),
    (oracle.MASK_CAUSAL, 1024, 1024),
    (oracle.MASK_CAUSAL, 300, 300),
    (oracle.MASK_CAUSAL, 200, 333),
    (oracle.MASK_CAUSAL, 333, 200),
    (oracle.MASK_CAUSAL, 1, 1),
]


@pytest.mark.parametrize("case", PLAN_CASES)
def test_plan_is_a_valid_schedule(case):
    kind, Nq, Nkv = case
    qt, kt = eio.plan(kind, None, Nq, Nkv)
    assert oracle.check_schedule(kind, None, Nq, Nkv, qt, kt) == 0
    assert np.all(kt[:, 1] % 16 == 0) and np.all(kt[:, 1] <= 128) and np.all(qt[:, 1] <= 128)


@pytest.mark.parametrize("seed", range(6))
def test_plan_block_maps_valid_and_predicate_free(seed):
    rng = np.random.default_rng(10 + seed)
    Nq, Nkv = int(rng.integers(1, 600)), int(rng.integers(1, 600))
    bm = _random_map(rng, (Nq + 15) // 16, (Nkv + 15) // 16, rng.uniform(0.05, 0.95))
    if seed % 2:
        bm = np.repeat(bm[::4], 4, axis=0)[: bm.shape[0]]  # runs of identical rows
    qt, kt = eio.plan(oracle.MASK_BLOCK, bm, Nq, Nkv)
    assert oracle.check_schedule(oracle.MASK_BLOCK, bm, Nq, Nkv, qt, kt) == 0
    # only a tile running past Nkv may need a predicate
    for c0, nc, part in kt:
        assert part == (1 if c0 + nc > Nkv else 0)
    # Q tiles start on 16-row boundaries and span a multiple of 16 rows unless
    # they end at Nq (the d=64 epilogue stores O in 16-row boxes)
    for r0, nr, _, _ in qt:
        assert r0 % 16 == 0 and (nr % 16 == 0 or r0 + nr == Nq)


def test_plan_frame_config_has_no_partial_tiles():
    bm = eio.frame_block_map(24, 1040)
    qt, kt = eio.plan(oracle.MASK_BLOCK, bm, 24960, 24960)
    assert oracle.check_schedule(oracle.MASK_BLOCK, bm, 24960, 24960, qt, kt) == 0
    assert kt[:, 2].sum() == 0
    assert len(qt) == 24 * 9  # 8 tiles of 128 rows and one of 16 per 1040-row frame
    # live (query row, key) pairs visited == allowed pairs: nothing padded on the key side
    visited = sum(int(r[1]) * int(kt[r[2]:r[2] + r[3], 1].sum()) for r in qt)
    assert visited == 69 * 1040 * 1040


@pytest.mark.parametrize("Nq,Nkv", [(1, 1), (300, 300), (1000, 77), (77, 1000), (4097, 4097)])
def test_plan_q_tiles_on_16_row_boundaries(Nq, Nkv):
    for kind in (oracle.MASK_NONE, oracle.MASK_CAUSAL):
        qt, kt = eio.plan(kind, None, Nq, Nkv)
        assert oracle.check_schedule(kind, None, Nq, Nkv, qt, kt) == 0
        for r0, nr, _, _ in qt:
            assert r0 % 16 == 0 and (nr % 16 == 0 or r0 + nr == Nq)


def test_plan_causal_counts():
    qt, kt = eio.plan(oracle.MASK_CAUSAL, None, 16384, 16384)
    assert len(qt) == 128 and len(kt) == 128 * 129 // 2
    assert kt[:, 2].sum() == 128  # one diagonal tile per Q tile


# ---------------------------------------------------------------- errors
FAKE = 0x10000  # never dereferenced: every case fails validation first


def _fwd(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Hq=2, Hkv=2, Nq=16, Nkv=16, d=64,
                scale=0.125, mask=0, bm=None, dtype=0, stream=None)
    args.update(kw)
    return eio.lib().attn_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"],
                              args["Hq"], args["Hkv"], args["Nq"], args["Nkv"], args["d"],
                              args["scale"], args["mask"], args["bm"], args["dtype"], args["stream"])


def test_argument_errors():
    assert _fwd(q=None) == 1
    assert _fwd(Hq=3, Hkv=2) == 2
    assert _fwd(Nq=0) == 2
    assert _fwd(scale=0.0) == 2
    assert _fwd(scale=float("nan")) == 2
    assert _fwd(q=FAKE + 8) == 3
    assert _fwd(d=96) == 4
    assert _fwd(dtype=7) == 4
    assert _fwd(mask=2) == 5
    assert _fwd(mask=9) == 5
    L = eio.lib()
    assert L.attn_decode(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 12, 4, 64, 128, 0.1, None) == 4  # G = 3
    assert L.attn_decode(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 8, 4, 64, 96, 0.1, None) == 4
    assert L.attn_decode(FAKE, FAKE, FAKE, None, FAKE, None, 1, 8, 4, 64, 128, 0.1, None) == 1
    assert L.attn_decode(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 8, 4, 0, 128, 0.1, None) == 2
    assert L.attn_classify(0, None, 10, 10, 0, 16, FAKE) == 2
    assert L.attn_classify(2, None, 10, 10, 16, 16, FAKE) == 5


def test_last_error_detail_text():
    assert _fwd(q=FAKE + 4) == 3
    assert "aligned" in eio.last_error()
    assert _fwd(Hq=3, Hkv=2) == 2
    assert "multiple" in eio.last_error()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_no_device_is_an_error_not_a_crash():
    # valid arguments, no GPU: reported as a CUDA error, nothing dereferenced
    assert _fwd() == 6
    assert eio.lib().attn_shutdown() == 0


def test_backward_bound_and_stats_argument_errors():
    """attn_bwd, attn_key_stats and attn_fwd_bound reject bad arguments on the
    host, before any device work (their status codes as documented)."""
    L = eio.lib()

    def bwd(mask=0, bm=None, d=64, q=FAKE, Hq=2, Hkv=2):
        return L.attn_bwd(q, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, Hq, Hkv, 16, 16, d, 0.125, mask,
                          bm, None)
    assert bwd(q=None) == 1
    assert bwd(Hq=3) == 2
    assert bwd(d=96) == 4
    assert bwd(mask=2, bm=None) == 5  # BLOCK without its map
    assert bwd(mask=9) == 5
    assert L.attn_key_stats(None, FAKE, FAKE, 1, 16, 2, 64, None) == 1
    assert L.attn_key_stats(FAKE, FAKE, FAKE, 1, 0, 2, 64, None) == 2
    assert L.attn_key_stats(FAKE, FAKE, FAKE, 1, 16, 2, 96, None) == 4
    assert L.attn_key_stats(FAKE + 8, FAKE, FAKE, 1, 16, 2, 64, None) == 3

    def fb(kbar=FAKE, radius=FAKE, nfb=None, d=64, mask=0, bm=None, o=FAKE):
        return L.attn_fwd_bound(FAKE, FAKE, FAKE, o, None, 1, 2, 2, 16, 16, d, 0.125, mask, bm, kbar, radius, nfb,
                                None)
    assert fb(kbar=None) == 1
    assert fb(o=None) == 1
    assert fb(d=32) == 4
    assert fb(mask=2) == 5
    assert fb(kbar=FAKE + 4) == 3
    assert fb(nfb=FAKE + 2) == 3


# ------------------------------------------------------- binding checks
def test_binding_rejects_block_maps_of_the_wrong_size():
    """The library reads ceil(Nq/16) x ceil(Nkv/16) bytes of the map: the
    binding refuses any other shape instead of letting it read past the end."""
    bm = np.ones((3, 4), np.uint8)
    qt, _ = eio.plan(oracle.MASK_BLOCK, bm, 48, 64)  # 3 x 4 blocks: accepted
    assert len(qt) == 1
    for Nq, Nkv in [(49, 64), (48, 65), (32, 64), (48, 48)]:
        with pytest.raises(ValueError, match="block_map"):
            eio.plan(oracle.MASK_BLOCK, bm, Nq, Nkv)
        with pytest.raises(ValueError, match="block_map"):
            eio.classify(oracle.MASK_BLOCK, bm, Nq, Nkv, 16, 16)


def test_binding_rejects_host_tensors():
    """Device entry points take CUDA tensors only; a host tensor is refused
    before any pointer reaches the library."""
    import torch
    x = torch.zeros(1, 16, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        eio.attn_fwd(x, x, x)
    with pytest.raises(ValueError, match="CUDA"):
        eio.attn_bwd(x, x, x, x, torch.zeros(1, 2, 16), x)
    with pytest.raises(ValueError, match="CUDA"):
        eio.key_stats(x)
    with pytest.raises(ValueError, match="CUDA"):
        eio.attn_decode(x[0], x, x, torch.zeros(1, dtype=torch.int32))


def test_bench_plan_statistics():
    """The tile-plan figures the bench line carries (host only): causal
    counts in closed form; on the frame mask the plan has no partial tile,
    where a plain 128 x 128 grid has 818 partial among 5023 live ones."""
    import bench
    g = bench.plan_stats(bench.WORKLOADS["gpt2"])
    assert (g["q_tiles"], g["kv_tile_visits"], g["partial_visits"]) == (8, 36, 8)
    lg = bench.plan_stats(bench.WORKLOADS["long"])
    assert (lg["q_tiles"], lg["kv_tile_visits"], lg["partial_visits"]) == (128, 128 * 129 // 2, 128)
    f = bench.plan_stats(bench.WORKLOADS["frame"])
    assert f["q_tiles"] == 24 * 9 and f["partial_visits"] == 0 and f["partial_share"] == 0.0
    assert (f["grid128_live"], f["grid128_partial"]) == (4205 + 818, 818)


def test_error_detail_is_per_thread_and_host_calls_are_thread_safe():
    """attn_last_error_detail reports the calling thread's own last failure
    while other threads fail differently at the same time (ctypes releases
    the GIL during the calls); concurrent host-only planning gives the same
    plans as serial planning."""
    import threading
    L = eio.lib()
    errors = []

    def failing(kind):
        buf = ctypes.create_string_buffer(256)
        for _ in range(2000):
            rc = _fwd(q=None) if kind == "null" else _fwd(Hq=3, Hkv=2)
            L.attn_last_error_detail(buf, 256)
            text = buf.value.decode()
            if (kind == "null" and (rc != 1 or "non-NULL" not in text)) or \
               (kind == "shape" and (rc != 2 or "multiple" not in text)):
                errors.append((kind, rc, text))
                return

    rng = np.random.default_rng(99)
    maps = [(int(n), int(m), _random_map(rng, (int(n) + 15) // 16, (int(m) + 15) // 16, 0.5))
            for n, m in rng.integers(1, 900, size=(8, 2))]
    serial = [eio.plan(oracle.MASK_BLOCK, bm, n, m) for n, m, bm in maps]
    planned = [None] * len(maps)

    def planning(i):
        n, m, bm = maps[i]
        for _ in range(20):
            planned[i] = eio.plan(oracle.MASK_BLOCK, bm, n, m)

    threads = [threading.Thread(target=failing, args=(k,)) for k in ("null", "shape", "null", "shape")]
    threads += [threading.Thread(target=planning, args=(i,)) for i in range(len(maps))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors[:3]
    for (qs, ks), (qp, kp) in zip(serial, planned):
        assert np.array_equal(qs, qp) and np.array_equal(ks, kp)


def test_io_complexity_worked_example(golden):
    """bench.io_elements against the FlashAttention page's section-5 numbers:
    standard attention ~N^2 element accesses, the tiled kernel ~N^2 d^2 / M."""
    import bench
    g = golden("io_complexity_flashattention_sec5.txt")
    std, tiled = bench.io_elements(int(g["N"]), int(g["d"]), g["M"])
    assert round(std / 1e4) == g["standard_1e4"]
    assert round(tiled / 1e4, 1) == g["tiled_1e4"]
    assert round(std / tiled) == g["ratio"]


def test_kv_cache_and_attention_matrix_worked_examples(golden):
    """bench's size helpers against the pages' worked numbers: the inference
    page's KV cache example (per token, for 128 users x 2048 tokens, and with
    MQA's single KV head) and the FlashAttention page's size of S."""
    import bench
    g = golden("kv_cache_size_inference_page.txt")
    per = bench.kv_cache_bytes_per_token(int(g["layers"]), int(g["heads"]), int(g["head_dim"]))
    assert per == g["bytes_per_token"] and per / 2 ** 20 == g["mb_per_token"]
    total = per * int(g["users"]) * int(g["tokens"])
    assert total / 2 ** 30 == g["gb_total"]
    mqa = bench.kv_cache_bytes_per_token(int(g["layers"]), 1, int(g["head_dim"])) * int(g["users"]) * int(g["tokens"])
    assert mqa / 2 ** 30 == g["gb_total_mqa"]
    s = golden("attention_matrix_size_flashattention_sec1.txt")
    n = bench.attention_matrix_elements(int(s["N"]), int(s["heads"]), int(s["batch"]))
    assert round(n / 1e8, 1) == s["elements_1e8"] and round(2 * n / 1e9, 1) == s["gb_16bit"]

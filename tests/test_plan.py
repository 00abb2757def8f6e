"""The library's launch plans (sparse_query_attention_b200/csrc/sqa_plan.h),
compiled with g++ on the CPU and checked against their stated rules: tile
packing, the GEMM raster, the decode chunking, the forward's cover of its
query tiles and the cluster split of a long reduction."""

import ctypes
import itertools
import os
import random
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_query_attention_b200", "csrc")


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not found")
    out = str(tmp_path_factory.mktemp("plan") / "libplan.so")
    subprocess.run([gxx, "-std=c++17", "-O1", "-shared", "-fPIC", "-I", CSRC,
                    os.path.join(ROOT, "tests", "plan_harness.cpp"), "-o", out], check=True)
    h = ctypes.CDLL(out)
    h.h_fwd_wave_plan.argtypes = [ctypes.c_longlong, ctypes.c_longlong, ctypes.c_longlong, ctypes.c_int,
                                  ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
    h.h_cluster_split.argtypes = [ctypes.c_longlong, ctypes.c_longlong, ctypes.c_longlong, ctypes.c_int,
                                  ctypes.POINTER(ctypes.c_int)]
    return h


def decode_plan(lib, B, H_q, H_kv, L):
    out = (ctypes.c_int * 5)()
    lib.h_decode_plan(B, H_q, H_kv, L, out)
    return dict(zip(["g", "log2g", "n_sub", "chunk", "n_split"], out))


def fwd_plan(lib, n_tblk, yz, n_tiles, sms, masked=False):
    out = (ctypes.c_int * 2)()
    lib.h_fwd_wave_plan(n_tblk, yz, n_tiles, sms, int(masked), out)
    return ["two-tile", "split", "mixed"][out[0]], out[1]


def cluster_split(lib, units, work, min_work, max_split, max_clusters):
    arr = (ctypes.c_int * 5)(*max_clusters)
    return lib.h_cluster_split(units, work, min_work, max_split, arr)


def test_head_pack_is_the_largest_power_of_two_dividing_g(lib):
    for G in range(1, 400):
        g = lib.h_head_pack(G)
        assert g & (g - 1) == 0 and G % g == 0 and g <= 128
        assert g == 128 or G % (2 * g) != 0


def test_gemm_raster_keeps_the_smaller_operand_resident(lib):
    assert lib.h_gemm_group_m(32768, 4096, 4096, 256) == 1      # W (32 MB) stays: N fastest
    assert lib.h_gemm_group_m(8192, 8192, 8192, 256) == 8       # both 128 MB: groups of 8 row tiles
    assert lib.h_gemm_group_m(512, 50000, 4096, 256) == 2       # A (4 MB) stays: all row tiles, M fastest
    assert lib.h_gemm_group_m(300, 100, 64, 128) == 1           # tiny: B is the smaller operand
    assert lib.h_gemm_group_m(16384, 256, 256, 128) == 1


DECODE_SHAPES = list(itertools.product([1, 4, 16, 64], [(16, 16), (16, 4), (8, 4), (4, 4), (4, 1), (6, 2), (8, 8)],
                                       [1, 63, 64, 255, 256, 1000, 4097, 32768, 131072]))


@pytest.mark.parametrize("B,heads,L", DECODE_SHAPES)
def test_decode_chunks_cover_the_cache(lib, B, heads, L):
    H_q, H_kv = heads
    p = decode_plan(lib, B, H_q, H_kv, L)
    G = H_q // H_kv
    assert p["g"] == lib.h_head_pack(G) and p["n_sub"] * p["g"] == G and 1 << p["log2g"] == p["g"]
    assert p["chunk"] % 64 == 0 and p["chunk"] >= 64
    # every chunk holds keys, and together they cover [0, L)
    assert p["n_split"] * p["chunk"] >= L and (p["n_split"] - 1) * p["chunk"] < L
    # no more chunks than 256-key chunks would give
    assert p["n_split"] <= max(1, (L + 255) // 256)


def test_decode_long_caches_fill_two_waves(lib):
    slots = lib.h_decode_slots()
    for B, (H_q, H_kv) in itertools.product([1, 4, 16], [(16, 16), (16, 4), (8, 4), (4, 1)]):
        p = decode_plan(lib, B, H_q, H_kv, 32768)
        units = B * H_kv * p["n_sub"]
        assert units * p["n_split"] >= min(2 * slots, units * ((32768 + 255) // 256))


def test_forward_cover_of_the_bench_shapes(lib):
    # N = 32768, d = 128, 148 SMs.  SQA (8,4): 128-token blocks (g = 2), 4 CTAs per block.
    assert fwd_plan(lib, 256, 4, 512, 148) == ("two-tile", 0)
    # xSQA (4,4): 256-token blocks (g = 1); 444 two-tile CTAs fill 3 waves, the rest split.
    assert fwd_plan(lib, 128, 4, 256, 148) == ("mixed", 111)
    # MHA (16,16): 2048 CTAs, 13.8 waves: two-tile.
    assert fwd_plan(lib, 128, 16, 256, 148)[0] == "two-tile"
    # masked problems keep the two-tile grid whatever the waves
    assert fwd_plan(lib, 128, 4, 256, 148, masked=True) == ("two-tile", 0)


def test_forward_cover_invariants(lib):
    rng = random.Random(7)
    for _ in range(2000):
        n_tblk = rng.randint(1, 600)
        yz = rng.randint(1, 64)
        n_tiles = 2 * n_tblk - rng.randint(0, 1)
        sms = rng.choice([132, 148, 160])
        cover, n_a = fwd_plan(lib, n_tblk, yz, n_tiles, sms)
        if cover == "mixed":
            assert 0 < n_a < n_tblk
            assert n_a * yz <= (n_tblk * yz // sms) * sms   # the two-tile part fits in whole waves
        else:
            assert n_a == 0


MAXC = [148, 74, 36, 16, 8]  # clusters of 1, 2, 4, 8, 16 CTAs running at once (one CTA per SM)


def test_cluster_split_examples(lib):
    assert cluster_split(lib, 8, 256, 4, 16, MAXC) == 16     # the layer's weight gradient: 8 tiles
    assert cluster_split(lib, 32, 256, 4, 16, MAXC) == 4     # 32 tiles: clusters of 8 would not all fit
    assert cluster_split(lib, 1, 20, 8, 8, MAXC) == 2        # work-limited
    assert cluster_split(lib, 100, 10**6, 4, 8, MAXC) == 1   # the grid already fills the device
    assert cluster_split(lib, 32, 256, 4, 8, MAXC) == 4      # key split of a 32-unit forward


def test_cluster_split_is_the_largest_that_qualifies(lib):
    rng = random.Random(11)
    for _ in range(3000):
        units = rng.randint(1, 200)
        work = rng.randint(1, 2000)
        min_work = rng.choice([4, 8])
        max_split = rng.choice([8, 16])
        c = cluster_split(lib, units, work, min_work, max_split, MAXC)
        ok = lambda k: work >= min_work * k and units <= MAXC[k.bit_length() - 1]
        if c > 1:
            assert ok(c)
        bigger = [k for k in (2, 4, 8, 16) if c < k <= max_split]
        assert not any(ok(k) for k in bigger)

"""Host logic of the GEMM dispatch, on the CPU (no device is touched): the
tile configuration the cost model picks, and the CTA-pair GEMM's plan for the
tiles past its last full wave (the decisions for the workloads' shapes, and
the invariants every plan keeps: the split ranges cover K with none empty,
only the ragged last wave is split or halved, the scratch slots and counters
suffice)."""

import ctypes

import pytest

import fp8_w8a8_static_b200 as fw

PAIRS = 74  # CTA pairs resident at once on a 148-SM B200


def test_two_tower_down_projection():
    """Both towers' down projections (192 + 48 tiles, K = 12288): three full
    waves, then the 18 remaining tiles split four ways."""
    assert fw.split_plan(240, PAIRS, 96) == dict(dp_tiles=222, split_tiles=18, splits=4,
                                                 kb_per_split=24, halves=1)


def test_short_k_tail_runs_as_halves():
    """The shared-quant Q/K/V launch (160 tiles, K = 3072, 24 K steps): too
    short to split over K; the 12 tiles past the second wave run as 24
    256x128 halves, with or without scratch."""
    want = dict(dp_tiles=148, split_tiles=12, splits=1, kb_per_split=24, halves=2)
    assert fw.split_plan(160, PAIRS, 24) == want
    assert fw.split_plan(160, PAIRS, 24, scratch=False) == want


def test_long_k_without_scratch_runs_halves():
    """Without scratch a long-K remainder cannot split over K; 18 tiles fill
    less than half a wave, so they run as halves."""
    assert fw.split_plan(240, PAIRS, 96, scratch=False) == dict(
        dp_tiles=222, split_tiles=18, splits=1, kb_per_split=96, halves=2)


def test_remainder_over_half_a_wave_runs_whole():
    """128 tiles (c1 1024x8192 and 4096x2048 at K = 2048): 54 remain past the
    first wave; as halves they would be 108 units, two half-waves, no faster
    than one whole wave, so they run whole."""
    assert fw.split_plan(128, PAIRS, 16) == dict(dp_tiles=128, split_tiles=0, splits=1,
                                                 kb_per_split=16, halves=1)
    assert fw.split_plan(37 + PAIRS, PAIRS, 16)["halves"] == 2   # 37: exactly half a wave
    assert fw.split_plan(38 + PAIRS, PAIRS, 16)["halves"] == 1


def test_single_partial_wave_runs_halves():
    """Fewer tiles than pairs (c1 256x2048: 8 tiles): every tile is cut in
    two, so twice as many SMs share the work."""
    assert fw.split_plan(8, PAIRS, 16) == dict(dp_tiles=0, split_tiles=8, splits=1,
                                               kb_per_split=16, halves=2)


def test_threshold_at_64_k_steps():
    assert fw.split_plan(10, PAIRS, 63)["splits"] == 1
    assert fw.split_plan(10, PAIRS, 64)["splits"] > 1


def test_threshold_at_ragged_k():
    """The threshold counts 128-byte K steps, ceil(K / 128): K = 8064 is 63
    steps (not split), K = 8080 (a multiple of 16 below 8192) is already 64
    steps and splits like K = 8192."""
    assert fw.split_plan(10, PAIRS, -(-8064 // 128))["splits"] == 1
    assert -(-8080 // 128) == 64
    p = fw.split_plan(10, PAIRS, -(-8080 // 128))
    assert p == fw.split_plan(10, PAIRS, 8192 // 128) and p["splits"] > 1


def test_ragged_k_case_of_the_gpu_tests():
    """M=300, N=520, K=8208: 6 tiles, 65 K steps (the last one partial)."""
    assert fw.split_plan(6, PAIRS, 65) == dict(dp_tiles=0, split_tiles=6, splits=4,
                                               kb_per_split=17, halves=1)


def test_full_waves_are_not_split():
    for waves in (1, 2, 3):
        p = fw.split_plan(waves * PAIRS, PAIRS, 96)
        assert p["splits"] == 1 and p["halves"] == 1 and p["dp_tiles"] == waves * PAIRS


@pytest.mark.parametrize("pairs", [1, 2, 37, PAIRS])
@pytest.mark.parametrize("scratch", [True, False])
def test_plan_invariants(pairs, scratch):
    for tiles in range(0, 400, 7):
        for num_kb in (1, 2, 9, 24, 63, 64, 65, 96, 97, 512):
            p = fw.split_plan(tiles, pairs, num_kb, scratch)
            dp, st, s, kbs, h = (p["dp_tiles"], p["split_tiles"], p["splits"], p["kb_per_split"],
                                 p["halves"])
            assert dp + st == tiles and 1 <= s <= 4 and h in (1, 2)
            assert s == 1 or h == 1                            # a K split or halves, not both
            if s == 1 and h == 1:
                assert st == 0 and kbs == num_kb
                continue
            assert dp % pairs == 0 and st == tiles % pairs    # only the ragged last wave
            if h == 2:
                assert 2 * st <= pairs and kbs == num_kb       # halves fill one wave at most
                assert not (scratch and num_kb >= 64 and st <= 128 and s > 1)
                continue
            assert scratch and num_kb >= 64
            assert (s - 1) * kbs < num_kb <= s * kbs           # covers K, no empty range
            assert kbs >= 2
            assert st * s <= min(2 * pairs, 148)               # scratch slots
            assert st <= 128                                   # split-K counters


def test_argument_errors():
    lib = fw.load()
    out = [ctypes.c_int() for _ in range(5)]
    refs = [ctypes.byref(o) for o in out]
    assert lib.fp8ws_split_plan(10, PAIRS, 96, 1, None, *refs[1:]) == fw.ERR_NULL
    assert lib.fp8ws_split_plan(10, PAIRS, 96, 1, *refs[:4], None) == fw.ERR_NULL
    assert lib.fp8ws_split_plan(-1, PAIRS, 96, 1, *refs) == fw.ERR_SHAPE
    assert lib.fp8ws_split_plan(10, 0, 96, 1, *refs) == fw.ERR_SHAPE
    assert lib.fp8ws_split_plan(10, PAIRS, 0, 1, *refs) == fw.ERR_SHAPE


# ------------------------------------------------------- GEMM tile choice


def test_gemm_plan_workload_shapes_use_cta_pairs():
    """Every GEMM of the workloads runs on CTA pairs (c0, c1, c3 grouped, c4)."""
    shapes = [[(64, 704)], [(64, 256)]]
    shapes += [[(m, n)] for m in (256, 1024, 4096) for n in (2048, 8192)]
    shapes += [[(2048, 3072), (2048, 1024), (2048, 1024)]]
    shapes += [[(4096, 12288), (1024, 12288)], [(4096, 3072), (1024, 3072)]]
    for s in shapes:
        assert fw.gemm_plan(s) == "pair256", s


def test_gemm_plan_one_cta_tiles_when_pairs_need_an_extra_wave():
    """Model (per-SM output area per wave / efficiency): M=1, N=19008 is 75
    pair tiles, two waves on 74 pairs: 2 * 128*256 / 1.0 = 65536; as 75 one-CTA
    128x256 tiles it is one wave on 148 SMs: 128*256 / 0.85 = 38550, the
    smallest (128x128: 149 tiles, 2 * 16384 / 0.45 = 72818; 128x64: 297 tiles,
    3 * 8192 / 0.25 = 98304).  At N=18944 (74 pair tiles, one wave) the pair
    kernel's 32768 wins."""
    assert fw.gemm_plan([(1, 19008)]) == "cta256"
    assert fw.gemm_plan([(1, 18944)]) == "pair256"


def test_gemm_plan_argument_errors():
    lib = fw.load()
    M = (ctypes.c_int64 * 3)(64, 64, 64)
    N = (ctypes.c_int64 * 3)(256, 256, 256)
    cfg = ctypes.c_int()
    assert lib.fp8ws_gemm_plan(148, PAIRS, M, N, 1, None) == fw.ERR_NULL
    assert lib.fp8ws_gemm_plan(148, PAIRS, None, N, 1, ctypes.byref(cfg)) == fw.ERR_NULL
    for args in ((0, PAIRS, 1), (148, 0, 1), (148, PAIRS, 0), (148, PAIRS, 4)):
        sms, pairs, count = args
        assert lib.fp8ws_gemm_plan(sms, pairs, M, N, count, ctypes.byref(cfg)) == fw.ERR_SHAPE
    bad = (ctypes.c_int64 * 1)(0)
    assert lib.fp8ws_gemm_plan(148, PAIRS, M, bad, 1, ctypes.byref(cfg)) == fw.ERR_SHAPE
    assert lib.fp8ws_gemm_plan(148, PAIRS, M, N, 3, ctypes.byref(cfg)) == fw.OK
    assert cfg.value == 1

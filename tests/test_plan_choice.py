"""Host logic of the tensor-core conv's planner (choose_umma_config), no
GPU: a small C++ probe links libcc3d.so and reports the plan chosen for a
grid of shapes; the tests check the invariants every plan must satisfy
(shared and tensor memory within the SM's, N tiles that divide C_out,
weight slots of whole kernel rows, resident weights only where they are
valid) and the choices the design rests on (the residual block on CTA
pairs, the time_conv with resident weights)."""
import itertools
import os
import shutil
import subprocess

import pytest

from video_vae_causal_implicit_b200 import cc3d

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "video_vae_causal_implicit_b200", "csrc")
FIELDS = ("ok", "kc", "nt", "n_ntiles", "sub", "nbuf", "g_taps", "pair", "na", "nb",
          "tmem_cols", "ctas_per_sm", "params", "b_resident", "xs", "smem")
SMEM_MAX = 227 * 1024


def _cuda_include():
    for cand in (os.environ.get("CUDA_HOME"), "/usr/local/cuda"):
        if cand and os.path.exists(os.path.join(cand, "include", "cuda.h")):
            return os.path.join(cand, "include")
    return None


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    if not os.path.exists(cc3d.LIB_PATH):
        pytest.skip("libcc3d.so is not built")
    inc = _cuda_include()
    if inc is None or shutil.which("g++") is None:
        pytest.skip("needs g++ and the CUDA headers")
    exe = str(tmp_path_factory.mktemp("plan") / "plan_probe")
    libdir = os.path.dirname(cc3d.LIB_PATH)
    subprocess.run(["g++", "-O1", "-std=c++17", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                    "-I", inc, os.path.join(HERE, "plan", "plan_probe.cpp"), "-o", exe,
                    "-L", libdir, "-lcc3d", "-Wl,-rpath," + libdir], check=True)

    def run(cases):
        text = "\n".join(" ".join(str(int(v)) for v in c) for c in cases) + "\n"
        out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True).stdout
        return [dict(zip(FIELDS, map(int, line.split()))) for line in out.splitlines()]
    return run


def case(n=1, ci=64, co=64, h=30, w=52, kt=3, ks=3, rms=False, mt=1, sms=148, f8=False):
    return (n, ci, co, h, w, kt, ks, rms, mt, sms, f8)


GRID = [case(n=n, ci=ci, co=co, h=h, w=w, kt=kt, ks=ks, rms=rms, mt=mt)
        for (ci, co), (h, w), (kt, ks), rms, n, mt in itertools.product(
            [(32, 48), (64, 64), (96, 96), (96, 192), (192, 192), (192, 384), (384, 384)],
            [(9, 17), (30, 52), (120, 208), (240, 416)],
            [(3, 3), (3, 1), (1, 1)],
            [False, True], [1, 4], [1, 5])
        ]


def test_every_plan_fits_the_sm(probe):
    for c, p in zip(GRID, probe(GRID)):
        n, ci, co, h, w, kt, ks, rms, mt, sms, f8 = c
        assert p["ok"] == 1, c
        assert p["smem"] <= SMEM_MAX, (c, p)
        assert 32 <= p["tmem_cols"] <= 512 and p["tmem_cols"] & (p["tmem_cols"] - 1) == 0, (c, p)
        cta_sub = 1 if p["pair"] else p["sub"]
        assert p["tmem_cols"] >= p["nbuf"] * cta_sub * p["nt"], (c, p)
        assert co % p["nt"] == 0 and p["nt"] % 16 == 0, (c, p)
        assert p["n_ntiles"] * p["nt"] == co, (c, p)
        assert ci % p["kc"] == 0 and p["kc"] in (32, 64, 96), (c, p)
        if rms and co <= 256:
            assert p["nt"] == co and p["xs"] == 0, (c, p)  # the whole row
        elif rms:
            # a row wider than one MMA: its halves on the two CTAs of a
            # cluster, each with two accumulator buffers
            assert (p["xs"], p["nt"], p["n_ntiles"]) == (2, co // 2, 2), (c, p)
            assert p["pair"] == 0 and p["sub"] == 1 and p["nbuf"] == 2, (c, p)
        else:
            assert p["xs"] == 0, (c, p)
        assert p["params"] == co * (3 if rms else 1), (c, p)
        assert p["nt"] <= 256, (c, p)
        assert 1 <= p["ctas_per_sm"] <= 2, (c, p)


def test_slots_pair_and_resident_only_where_valid(probe):
    for c, p in zip(GRID, probe(GRID)):
        n, ci, co, h, w, kt, ks, rms, mt, sms, f8 = c
        # a weight slot holds one tap, or one whole kernel row of taps, or
        # (a 1 x 1 kernel with streamed weights) two channel chunks beside a
        # halo group of two slots
        if ks == 1 and p["g_taps"] == 2:
            assert not p["b_resident"] and (ci // p["kc"]) % 2 == 0 and p["na"] % 2 == 0, (c, p)
            assert p["na"] >= 4 and p["nb"] >= 3, (c, p)
        else:
            assert p["g_taps"] in (1, ks), (c, p)
        if p["pair"]:
            assert p["kc"] == 64 and p["sub"] == 2 and p["ctas_per_sm"] == 1, (c, p)
        if p["b_resident"]:
            assert ks == 1 and p["n_ntiles"] == 1 and p["g_taps"] == 1, (c, p)
            assert p["nb"] == kt * ci // p["kc"] and p["na"] >= 3, (c, p)
        else:
            assert 2 <= p["na"] <= 8 and 2 <= p["nb"] <= 8, (c, p)
            if ks == 3:
                assert p["na"] == 2, (c, p)
                # kernel-row slots wherever two of them fit beside the two
                # halo stages: every 64-channel-chunk plan up to N = 192
                if p["kc"] == 64 and p["nt"] <= 192:
                    assert p["g_taps"] == 3, (c, p)


def test_plan_is_a_function_of_the_problem(probe):
    """Asking twice gives the same plan (no hidden state), and the plan
    depends on the largest call (max_t), not on anything per call."""
    a = probe(GRID[:64])
    b = probe(GRID[:64])
    assert a == b


def test_downsample_conv_plans(probe):
    """The stride-2 spatial conv plans the input's four stride-2 phases
    seen through 2 x 2 views over the output frame (kt = 4, ks = 2): one tap
    per weight slot, weights streamed, within the SM."""
    cases = [case(n=n, ci=ci, co=co, h=h, w=w, kt=4, ks=2, mt=mt)
             for (ci, co), (h, w), n, mt in itertools.product(
                 [(64, 64), (96, 96), (64, 128), (192, 192)],
                 [(10, 12), (15, 26), (48, 80), (240, 416)], [1, 2], [1, 17])]
    for c, p in zip(cases, probe(cases)):
        assert p["ok"] == 1 and p["smem"] <= SMEM_MAX and p["g_taps"] == 1, (c, p)
        assert p["b_resident"] == 0 and p["na"] == 2 and 2 <= p["nb"] <= 8, (c, p)


def test_fp8_plans(probe):
    """FP8 E4M3 operands: 128-channel chunks (one 128-byte swizzled row per
    pixel), on every tile shape that takes them, within the SM."""
    cases = [case(n=n, ci=ci, co=co, h=h, w=w, ks=ks, mt=mt, f8=True)
             for (ci, co), (h, w), ks, n, mt in itertools.product(
                 [(128, 128), (384, 384), (256, 512)], [(16, 20), (30, 52), (120, 208)],
                 [3, 1], [1, 2], [1, 5])]
    for c, p in zip(cases, probe(cases)):
        assert p["ok"] == 1 and p["kc"] == 128 and p["smem"] <= SMEM_MAX, (c, p)
    # channel counts that are not whole 128-channel chunks have no FP8 plan
    bad = probe([case(ci=96, co=96, f8=True), case(ci=192, co=192, f8=True)])
    assert [p["ok"] for p in bad] == [0, 0]


def test_the_documented_choices(probe):
    c4, tc192, tc384, c2 = probe([
        case(ci=192, co=192, h=240, w=416, rms=True, mt=9),
        case(ci=192, co=192, h=120, w=208, ks=1, mt=9),
        case(ci=384, co=384, h=60, w=104, ks=1, mt=5),
        case(ci=384, co=384, h=30, w=52, mt=5),
    ])
    # the residual block's convs run on CTA pairs with kernel-row weight slots
    assert (c4["pair"], c4["nt"], c4["g_taps"]) == (1, 192, 3)
    # the 192-channel time_conv keeps its weights resident; 384 channels do not fit
    assert (tc192["pair"], tc192["b_resident"], tc192["nb"]) == (1, 1, 9)
    assert tc384["b_resident"] == 0
    # the latent-resolution layer: kernel-row weight slots
    assert c2["g_taps"] == 3


@pytest.fixture(scope="module")
def deal(tmp_path_factory):
    if not os.path.exists(cc3d.LIB_PATH):
        pytest.skip("libcc3d.so is not built")
    inc = _cuda_include()
    if inc is None or shutil.which("g++") is None:
        pytest.skip("needs g++ and the CUDA headers")
    exe = str(tmp_path_factory.mktemp("deal") / "deal_probe")
    libdir = os.path.dirname(cc3d.LIB_PATH)
    subprocess.run(["g++", "-O1", "-std=c++17", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                    "-I", inc, os.path.join(HERE, "plan", "deal_probe.cpp"), "-o", exe,
                    "-L", libdir, "-lcc3d", "-Wl,-rpath," + libdir], check=True)

    def run(cases):
        text = "\n".join(" ".join(str(int(v)) for v in c) for c in cases) + "\n"
        out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True).stdout
        return [dict(zip(("ok", "plan", "one", "pair_plan", "pair_one"), map(int, line.split())))
                for line in out.splitlines()]
    return run


def dcase(n=1, ci=384, co=384, h=30, w=52, kt=3, ks=3, rms=False, mt=5, sms=148, t_out=5,
          cached=True, stride=1):
    return (n, ci, co, h, w, kt, ks, rms, mt, sms, t_out, cached, stride)


def test_call_cost_without_a_cache(deal):
    """A call without a cache skips its first frames' causal zero taps, so it
    costs less than the same call with one, and a call whose units all fit
    one wave costs one unit: all kt taps once some output frame reads no
    zero frame, one tap for a single uncached frame."""
    cases = [dcase(t_out=t, cached=c) for t in (1, 2, 3, 5) for c in (False, True)]
    res = deal(cases)
    for i in range(0, len(res), 2):
        unc, cac = res[i], res[i + 1]
        assert unc["ok"] == cac["ok"] == 1
        assert unc["plan"] <= cac["plan"] and unc["one"] <= cac["one"], cases[i]
    one_frame_unc, one_frame_cac = res[0], res[1]
    # one output frame, one wave: the plan tiles' unit with 1 of 3 taps live
    assert one_frame_cac["plan"] == 3 * one_frame_unc["plan"]


def test_uncached_whole_sequence_takes_the_pair_tiles(deal):
    """The 384-channel latent layer planned for 5 frames: its own tiles (one
    CTA per tile, one wave) for a 5-frame call with a cache; for the
    uncached whole-sequence call, the one-frame tiles (CTA pairs), whose
    six spare tiles are dealt to clusters that drew cheap first-frame tiles."""
    unc, cac = deal([dcase(cached=False), dcase(cached=True)])
    assert (unc["pair_plan"], unc["pair_one"]) == (0, 1)
    assert unc["one"] < unc["plan"]
    assert cac["one"] > cac["plan"]


def test_serpentine_deal_pairs_spare_units_with_cheap_ones(deal):
    """80 pair units on 74 clusters, dealt last frame first: 48 full units
    (3 live taps), 16 of frame 1 (2 taps), 16 of frame 0 (1 tap).  The
    serpentine deal gives the 6 spare frame-0 units to the clusters that
    drew frame-0 units in the first round, so the makespan is one full unit
    -- the cost of one cached frame, whose units all run at once.  A plain
    round-robin deal would give them to clusters with full units (4 taps)."""
    unc5, cac1 = deal([dcase(cached=False, t_out=5), dcase(cached=True, t_out=1)])
    assert (unc5["pair_one"], cac1["pair_one"]) == (1, 1)
    assert unc5["one"] == cac1["one"]

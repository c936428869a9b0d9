"""A fast cross-section of every kind of launch the library makes, each
checked against the fp64 oracle on a small case.  This file is collected
before the other GPU tests, so that a regression in one kind of plan names
that kind in the first failing test instead of hiding the rest of the
suite behind an unrelated one.  Each case asserts which kind of plan it
got through the plan's stats."""
import ctypes

import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, assert_close_fp32, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


def _shape(plan):
    st = plan.stats()
    return dict(variant=st.variant, mma_ctas=st.mma_ctas, tile_w=st.tile_w,
                resident=st.w_resident, n_tile=st.n_tile, k_split=st.k_split,
                row_ctas=st.row_ctas)


def _conv(n, cin, cout, t, h, w, k=(3, 3, 3), seed=0, stride_t=1, cache=False, **plan_kw):
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=seed)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t,
                     stride_t=stride_t, **plan_kw)
    x = to_dev(synth.ndhwc(case["x"]))
    c = synth.normal((n, cin, 2, h, w), seed + 40) if cache else None
    t_out = (t - 1) // stride_t + 1
    y = torch.empty((n, t_out, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y, cache_in=to_dev(synth.ndhwc(c)) if cache else None)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                               cache=c.double().numpy() if cache else None,
                               pad=(k[1] // 2, k[2] // 2), stride_t=stride_t)
    return plan, y, ref


# (name, conv args, expected plan fields)
CONVS = [
    ("single_cta_32ch_chunks", dict(n=1, cin=32, cout=48, t=2, h=12, w=20),
     dict(mma_ctas=1, tile_w=8, resident=0)),
    ("single_cta_96ch_slabs_with_cache", dict(n=2, cin=96, cout=96, t=2, h=12, w=20, cache=True),
     dict(mma_ctas=1, tile_w=8, resident=0)),
    ("two_subtiles", dict(n=8, cin=32, cout=48, t=1, h=20, w=150),
     dict(mma_ctas=1, tile_w=16, resident=0)),
    ("cta_pair_with_cache", dict(n=1, cin=64, cout=64, t=2, h=17, w=9, cache=True),
     dict(mma_ctas=2, tile_w=16, resident=0)),
    ("resident_weights_single", dict(n=2, cin=32, cout=64, t=2, h=12, w=40, k=(1, 1, 1)),
     dict(mma_ctas=1, resident=1)),
    ("resident_weights_pair", dict(n=1, cin=64, cout=64, t=3, h=20, w=36, k=(3, 1, 1)),
     dict(mma_ctas=2, resident=1)),
    ("temporal_stride_2", dict(n=1, cin=64, cout=64, t=5, h=12, w=20, stride_t=2),
     dict(k_split=1)),
]


@pytest.mark.parametrize("name,args,expect", CONVS, ids=[c[0] for c in CONVS])
def test_conv_plan_kind(name, args, expect):
    args = dict(args)
    plan, y, ref = _conv(seed=len(name), **args)
    got = _shape(plan)
    assert got["k_split"] == 1
    for key, val in expect.items():
        assert got[key] == val, f"{name}: plan {got}"
    assert_close_bf16(ncthw_np(y), ref, name)


def test_rms_epilogue_with_next_cache():
    """Bias + RMS_norm + SiLU epilogue on a CTA pair, with the output's
    two-frame history written by the same kernel."""
    n, cin, cout, t, h, w = 1, 64, 128, 2, 16, 20
    g = synth.uniform((cout,), 0.5, 1.5, 7)
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=8)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t,
                     epi=cc3d.EPI_BIAS_RMS_SILU, gamma=to_dev(g))
    assert _shape(plan)["mma_ctas"] == 2
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    nc_out = torch.empty((n, 2, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y, next_cache_out=nc_out)
    cc3d.sync_status()
    assert torch.equal(nc_out.cpu(), y.cpu())
    conv = oracle.round_bf16_array(
        oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy()))
    ref = oracle.rms_norm(conv, g.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "rms epilogue")


def test_rms_row_split_over_a_cluster():
    """A 320-channel RMS row: each CTA of a cluster takes 160 channels of
    the same pixels, and the two swap each row's partial sum of squares."""
    n, cin, cout, t, h, w = 1, 64, 320, 2, 16, 20
    g = synth.uniform((cout,), 0.5, 1.5, 10)
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=11)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t,
                     epi=cc3d.EPI_BIAS_RMS_SILU, gamma=to_dev(g))
    got = _shape(plan)
    assert (got["row_ctas"], got["n_tile"], got["mma_ctas"]) == (2, 160, 1), got
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    conv = oracle.round_bf16_array(
        oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy()))
    ref = oracle.rms_norm(conv, g.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "rms row split over a cluster")


def test_thin_first_layer():
    case = synth.conv_case(3, 96, 2, 20, 24, seed_base=9, x_dist="uniform")
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), h=20, w=24, max_t=2)
    assert _shape(plan)["variant"] == cc3d.VARIANT_THIN
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((1, 2, 20, 24, 96), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    assert_close_bf16(ncthw_np(y), ref, "thin")


def test_fp32_conv():
    case = synth.conv_case(16, 16, 3, 8, 8, dtype=torch.float32, seed_base=10)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), h=8, w=8, max_t=3, dtype=cc3d.FP32)
    assert _shape(plan)["variant"] == cc3d.VARIANT_FP32
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((1, 3, 8, 8, 16), dtype=torch.float32, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(case["x"], case["w"], case["b"].double().numpy())
    assert_close_fp32(ncthw_np(y), ref, "fp32")


def test_spatial_stride_2():
    n, c, t, h, w = 1, 96, 2, 16, 24
    x = synth.normal((n, c, t, h, w), 11)
    wt = synth.kaiming_uniform(c, c, (1, 3, 3), 12)
    b = synth.uniform((c,), -0.1, 0.1, 13)
    plan = cc3d.Plan(to_dev(wt), to_dev(b), n=n, h=h, w=w, max_t=t, pad=(0, 0), stride_hw=2)
    xd = to_dev(synth.ndhwc(x))
    y = torch.empty((n, t, h // 2, w // 2, c), dtype=torch.bfloat16, device="cuda")
    plan.forward(xd, y)
    cc3d.sync_status()
    ref = oracle.conv2d_frames(synth.ncthw_view(xd.cpu()), wt[:, :, 0], b.double().numpy(),
                               stride=(2, 2), pad=(0, 1, 0, 1))
    assert_close_bf16(ncthw_np(y), ref, "spatial stride 2")


def test_block_with_fused_shortcut():
    n, cin, cout, t, h, w = 1, 64, 128, 2, 16, 20
    c = synth.block_case(cin, t, h, w, n=n, seed_base=14)
    wts = dict(w1=synth.kaiming_uniform(cout, cin, (3, 3, 3), 15),
               b1=synth.uniform((cout,), -0.1, 0.1, 16), g1=c["g1"],
               w2=synth.kaiming_uniform(cout, cout, (3, 3, 3), 17),
               b2=synth.uniform((cout,), -0.1, 0.1, 18), g2=synth.uniform((cout,), 0.5, 1.5, 19),
               w_sc=synth.kaiming_uniform(cout, cin, (1, 1, 1), 20),
               b_sc=synth.uniform((cout,), -0.1, 0.1, 21))
    blk = cc3d.Block(**{k: to_dev(v) for k, v in wts.items()}, n=n, h=h, w=w, max_t=t)
    x = to_dev(synth.ndhwc(c["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    blk.forward(x, y)
    cc3d.sync_status()
    d = lambda v: v.double().numpy()  # noqa: E731
    ref = oracle.resblock(synth.ncthw_view(x.cpu()), wts["w1"], d(wts["b1"]), d(wts["g1"]),
                          wts["w2"], d(wts["b2"]), d(wts["g2"]), w_sc=wts["w_sc"],
                          b_sc=d(wts["b_sc"]))
    assert_close_bf16(ncthw_np(y), ref, "block with shortcut")


def test_noalloc_entry_point():
    n, cin, cout, t, h, w = 1, 64, 64, 2, 17, 9
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=22)
    x = to_dev(synth.ndhwc(case["x"]))
    wt, b = to_dev(case["w"]), to_dev(case["b"])
    d = cc3d.Desc()
    d.n, d.c_in, d.c_out, d.h, d.w, d.max_t = n, cin, cout, h, w, t
    d.kt = d.kh = d.kw = 3
    d.pad_h = d.pad_w = 1
    d.stride_t = d.stride_h = d.stride_w = d.dil_t = d.dil_h = d.dil_w = d.groups = 1
    d.dtype = cc3d.BF16
    d.weight, d.bias, d.epi = wt.data_ptr(), b.data_ptr(), cc3d.EPI_BIAS
    y = torch.full((n, t, h, w, cout), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = cc3d.cc3d_forward_noalloc(d, ctypes.c_void_p(x.data_ptr()), t, None,
                                   ctypes.c_void_p(y.data_ptr()), None, None, None, None,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == cc3d.OK, cc3d.cc3d_status_string(st)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    assert_close_bf16(ncthw_np(y), ref, "noalloc")

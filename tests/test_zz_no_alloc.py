"""cc3d_forward_noalloc: the conv entry point for callers that cannot call
cudaMalloc (their device memory comes from a fixed pool they manage, or an
allocation's implicit synchronisation is not acceptable where they call).
Its output must match the planned entry point (cc3d_plan_create +
cc3d_forward) on the same inputs, call after call, although all its calls
share one fixed scratch array inside the library.

This file is named so that pytest collects it last."""
import ctypes

import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


def _desc_for(plan_kwargs, weight, bias, gamma=None):
    """Same descriptor a Plan builds, pointing at the caller's tensors."""
    co, ci, kt, kh, kw = (int(s) for s in weight.shape)
    d = cc3d.Desc()
    d.n, d.c_in, d.c_out = 1, ci, co
    d.h, d.w, d.max_t = plan_kwargs["h"], plan_kwargs["w"], plan_kwargs["max_t"]
    d.kt, d.kh, d.kw, d.pad_h, d.pad_w = kt, kh, kw, kh // 2, kw // 2
    d.stride_t = d.stride_h = d.stride_w = d.dil_t = d.dil_h = d.dil_w = d.groups = 1
    d.dtype = cc3d.BF16
    d.weight = weight.data_ptr()
    d.bias = bias.data_ptr() if bias is not None else None
    d.epi = plan_kwargs.get("epi", cc3d.EPI_BIAS)
    d.gamma = gamma.data_ptr() if gamma is not None else None
    d.beta = None
    return d


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_planned_conv_on_two_calls_in_a_row():
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # call 1: 384 -> 384 with a bias and a cache (a small frame, two N
    # tiles); call 2: different weights, no bias (the scratch's zero bias
    # must be cleared), 96 -> 192; call 3: a frame large enough for the CTA
    # pair, whose weights the scratch holds as plain rows behind a tensor map.
    cases = [
        dict(cin=384, cout=384, t=2, h=30, w=52, bias=True, cache=True, seed=1),
        dict(cin=96, cout=192, t=3, h=21, w=17, bias=False, cache=False, seed=2),
        dict(cin=64, cout=64, t=2, h=96, w=96, bias=True, cache=True, seed=3),
    ]
    outs = []
    for cs in cases:
        case = synth.conv_case(cs["cin"], cs["cout"], cs["t"], cs["h"], cs["w"],
                               seed_base=cs["seed"])
        x = to_dev(synth.ndhwc(case["x"]))
        w = to_dev(case["w"])
        b = to_dev(case["b"]) if cs["bias"] else None
        cache = (to_dev(synth.ndhwc(synth.normal((1, cs["cin"], 2, cs["h"], cs["w"]), 40)))
                 if cs["cache"] else None)
        kw = dict(h=cs["h"], w=cs["w"], max_t=cs["t"])
        plan = cc3d.Plan(w, b, **kw)
        if cs["seed"] == 3:
            assert plan.stats().mma_ctas == 2
        y_ref = torch.empty((1, cs["t"], cs["h"], cs["w"], cs["cout"]), dtype=torch.bfloat16,
                            device="cuda")
        plan.forward(x, y_ref, cache_in=cache)
        y = torch.full_like(y_ref, float("nan"))
        cache_out = torch.empty((1, 2, cs["h"], cs["w"], cs["cin"]), dtype=torch.bfloat16,
                                device="cuda")
        d = _desc_for(kw, w, b)
        st = cc3d.cc3d_forward_noalloc(d, _p(x), cs["t"], _p(cache), _p(y), _p(cache_out), None,
                                       None, None, stream)
        assert st == cc3d.OK, cc3d.cc3d_status_string(st)
        cc3d.sync_status()
        assert torch.equal(y.cpu(), y_ref.cpu())  # same kernel and tiles: same bytes
        assert torch.equal(cache_out[:, -2:].cpu(), x[:, -2:].cpu())
        ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"],
                                   case["b"].double().numpy() if cs["bias"] else None,
                                   cache=synth.ncthw_view(cache.cpu()) if cache is not None
                                   else None)
        assert_close_bf16(ncthw_np(y), ref, f"noalloc call {cs} vs oracle")
        outs.append(y)
        plan.close()
    torch.cuda.synchronize()


def test_noalloc_matches_planned_time_conv_with_resident_weights():
    """Temporal stride 2 with kernel (3, 1, 1): the CTA pair with every
    weight stage resident in shared memory, as the planned call."""
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    c, t, h, w = 192, 17, 30, 52
    case = synth.conv_case(c, c, t, h, w, k=(3, 1, 1), seed_base=4)
    x = to_dev(synth.ndhwc(case["x"]))
    wt, b = to_dev(case["w"]), to_dev(case["b"])
    kw = dict(h=h, w=w, max_t=t)
    plan = cc3d.Plan(wt, b, stride_t=2, **kw)
    st = plan.stats()
    assert (st.w_resident, st.mma_ctas) == (1, 2)
    t_out = (t - 1) // 2 + 1
    y_ref = torch.empty((1, t_out, h, w, c), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y_ref)
    y = torch.full_like(y_ref, float("nan"))
    d = _desc_for(kw, wt, b)
    d.stride_t = 2
    res = cc3d.cc3d_forward_noalloc(d, _p(x), t, None, _p(y), None, None, None, None, stream)
    assert res == cc3d.OK, cc3d.cc3d_status_string(res)
    cc3d.sync_status()
    assert torch.equal(y.cpu(), y_ref.cpu())
    plan.close()


def test_noalloc_residual_and_rms_epilogues():
    """The residual epilogue, and the RMS_norm + SiLU epilogue with the
    output's two-frame history (next_cache_out after a carried
    next_cache_in), against the planned call and the oracle."""
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    n, c, h, w = 1, 64, 20, 36
    # residual: 2 frames
    case = synth.conv_case(c, c, 2, h, w, seed_base=5)
    x, wt, b = to_dev(synth.ndhwc(case["x"])), to_dev(case["w"]), to_dev(case["b"])
    res = to_dev(synth.ndhwc(synth.normal((n, c, 2, h, w), 51)))
    kw = dict(h=h, w=w, max_t=2, epi=cc3d.EPI_BIAS_RESIDUAL)
    plan = cc3d.Plan(wt, b, **kw)
    y_ref = torch.empty_like(res)
    plan.forward(x, y_ref, residual=res)
    y = torch.full_like(res, float("nan"))
    st = cc3d.cc3d_forward_noalloc(_desc_for(kw, wt, b), _p(x), 2, None, _p(y), None, _p(res),
                                   None, None, stream)
    assert st == cc3d.OK, cc3d.cc3d_status_string(st)
    cc3d.sync_status()
    assert torch.equal(y.cpu(), y_ref.cpu())
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    assert_close_bf16(ncthw_np(y), ref + ncthw_np(res), "noalloc residual vs oracle")
    plan.close()
    # RMS + SiLU: one-frame call carrying next_cache_in
    case = synth.conv_case(c, c, 1, h, w, seed_base=6)
    x, wt, b = to_dev(synth.ndhwc(case["x"])), to_dev(case["w"]), to_dev(case["b"])
    g = to_dev(synth.uniform((c,), 0.5, 1.5, 52))
    nc_in = to_dev(synth.ndhwc(synth.normal((n, c, 2, h, w), 53)))
    kw = dict(h=h, w=w, max_t=1, epi=cc3d.EPI_BIAS_RMS_SILU)
    plan = cc3d.Plan(wt, b, gamma=g, **kw)
    y_ref = torch.empty((n, 1, h, w, c), dtype=torch.bfloat16, device="cuda")
    nc_ref = torch.empty_like(nc_in)
    plan.forward(x, y_ref, next_cache_in=nc_in, next_cache_out=nc_ref)
    y = torch.full_like(y_ref, float("nan"))
    nc = torch.full_like(nc_in, float("nan"))
    st = cc3d.cc3d_forward_noalloc(_desc_for(kw, wt, b, g), _p(x), 1, None, _p(y), None, None,
                                   _p(nc_in), _p(nc), stream)
    assert st == cc3d.OK, cc3d.cc3d_status_string(st)
    cc3d.sync_status()
    assert torch.equal(y.cpu(), y_ref.cpu())
    assert torch.equal(nc.cpu(), nc_ref.cpu())
    assert torch.equal(nc[:, :1].cpu(), nc_in[:, 1:].cpu())
    assert torch.equal(nc[:, 1:].cpu(), y.cpu())
    conv = oracle.round_bf16_array(
        oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy()))
    ref = oracle.rms_norm(conv, synth.uniform((c,), 0.5, 1.5, 52).double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "noalloc rms vs oracle")
    plan.close()


def test_noalloc_refuses_weights_beyond_its_scratch():
    big = torch.empty((512, 512, 3, 3, 3), dtype=torch.bfloat16, device="cuda")  # 14 MB
    d = _desc_for(dict(h=8, w=8, max_t=1), big, None)
    x = torch.zeros((1, 1, 8, 8, 512), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((1, 1, 8, 8, 512), dtype=torch.bfloat16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    launches = cc3d.cc3d_launch_count()
    st = cc3d.cc3d_forward_noalloc(d, _p(x), 1, None, _p(y), None, None, None, None, stream)
    assert st == cc3d.ERR_TOO_LARGE
    assert cc3d.cc3d_launch_count() == launches

"""cc3d_forward_host: convs whose x and y live in host memory, uploads and
downloads overlapped with the convs through the plan's three staging slots.
Every call's y must equal, byte for byte, the device-pointer call on the
same input (same kernel, same tiles), across more calls than slots (so the
slots are reused), for whole sequences and streamed one-frame chunks with
device caches, for the residual epilogue, the thin RGB conv, FP8 codes and
pageable host memory; and a whole sequence is checked against the oracle."""
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


def _pinned(t):
    return t.cpu().pin_memory()


def test_host_calls_equal_device_calls_whole_and_streamed():
    n, c, t, h, w = 1, 64, 4, 20, 36
    case = synth.conv_case(c, c, t, h, w, seed_base=60)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t)
    x = to_dev(synth.ndhwc(case["x"]))
    # device reference: the whole sequence, then one-frame chunks with caches
    y_ref = torch.empty((n, t, h, w, c), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y_ref)
    caches_ref = [torch.empty((n, 2, h, w, c), dtype=torch.bfloat16, device="cuda")
                  for _ in range(t)]
    ys_ref, cache = [], None
    for s in range(t):
        yc = torch.empty((n, 1, h, w, c), dtype=torch.bfloat16, device="cuda")
        plan.forward(x[:, s:s + 1].contiguous(), yc, cache_in=cache, cache_out=caches_ref[s])
        cache = caches_ref[s]
        ys_ref.append(yc)
    cc3d.sync_status()
    # host calls: the same five calls in one cc3d_forward_host (five calls,
    # three slots: two of them serve two calls)
    x_host = _pinned(x)
    frames = [_pinned(x[:, s:s + 1].contiguous()) for s in range(t)]
    y_host = torch.empty((n, t, h, w, c), dtype=torch.bfloat16).pin_memory()
    ys_host = [torch.empty((n, 1, h, w, c), dtype=torch.bfloat16).pin_memory() for _ in range(t)]
    caches = [torch.empty((n, 2, h, w, c), dtype=torch.bfloat16, device="cuda") for _ in range(t)]
    calls = [dict(x_host=x_host, y_host=y_host)]
    for s in range(t):
        calls.append(dict(x_host=frames[s], y_host=ys_host[s],
                          cache_in=caches[s - 1] if s > 0 else None, cache_out=caches[s]))
    plan.forward_host(calls)
    torch.cuda.current_stream().synchronize()
    cc3d.sync_status()
    assert torch.equal(y_host, y_ref.cpu())
    for s in range(t):
        assert torch.equal(ys_host[s], ys_ref[s].cpu()), s
        assert torch.equal(caches[s].cpu(), caches_ref[s].cpu()), s
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    assert_close_bf16(ncthw_np(y_host), ref, "host-buffer whole sequence vs oracle")
    # a second batch on the same plan reuses its slots and streams
    y2 = torch.empty_like(y_host).pin_memory()
    plan.forward_host([dict(x_host=x_host, y_host=y2)])
    torch.cuda.current_stream().synchronize()
    assert torch.equal(y2, y_ref.cpu())
    plan.close()


def test_host_calls_residual_thin_fp8_and_pageable():
    # residual epilogue (the residual stays on the device)
    n, c, t, h, w = 1, 96, 2, 17, 30
    case = synth.conv_case(c, c, t, h, w, seed_base=61)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t,
                     epi=cc3d.EPI_BIAS_RESIDUAL)
    x = to_dev(synth.ndhwc(case["x"]))
    res = to_dev(synth.ndhwc(synth.normal((n, c, t, h, w), 62)))
    y_ref = torch.empty_like(res)
    plan.forward(x, y_ref, residual=res)
    y_host = torch.empty(tuple(res.shape), dtype=torch.bfloat16)  # pageable
    plan.forward_host([dict(x_host=x.cpu(), y_host=y_host, residual=res)])
    torch.cuda.current_stream().synchronize()
    cc3d.sync_status()
    assert torch.equal(y_host, y_ref.cpu())
    plan.close()
    # the thin RGB first layer (its x has 3 channels per pixel)
    c3 = synth.conv_case(3, 96, 3, 20, 24, seed_base=63, x_dist="uniform")
    p3 = cc3d.Plan(to_dev(c3["w"]), to_dev(c3["b"]), h=20, w=24, max_t=3)
    x3 = to_dev(synth.ndhwc(c3["x"]))
    y3 = torch.empty((1, 3, 20, 24, 96), dtype=torch.bfloat16, device="cuda")
    p3.forward(x3, y3)
    y3h = torch.empty((1, 3, 20, 24, 96), dtype=torch.bfloat16).pin_memory()
    p3.forward_host([dict(x_host=_pinned(x3), y_host=y3h)])
    torch.cuda.current_stream().synchronize()
    cc3d.sync_status()
    assert torch.equal(y3h, y3.cpu())
    p3.close()
    # FP8 E4M3 codes in host memory
    c8 = synth.conv_case(128, 128, 2, 12, 20, seed_base=64)
    s_w = (c8["w"].float().abs().reshape(128, -1).max(dim=1).values / 448.0).contiguous()
    s_x = float(c8["x"].float().abs().max()) / 448.0
    p8 = cc3d.Plan(to_dev(c8["w"]), to_dev(c8["b"]), h=12, w=20, max_t=2, dtype=cc3d.FP8_E4M3,
                   w_scale=to_dev(s_w), x_scale=s_x)
    xb = to_dev(synth.ndhwc(c8["x"]))
    q = torch.empty(xb.shape, dtype=torch.uint8, device="cuda")
    cc3d.quantize_e4m3(xb, s_x, q)
    y8 = torch.empty((1, 2, 12, 20, 128), dtype=torch.bfloat16, device="cuda")
    p8.forward(q, y8)
    y8h = torch.empty((1, 2, 12, 20, 128), dtype=torch.bfloat16).pin_memory()
    p8.forward_host([dict(x_host=_pinned(q), y_host=y8h)])
    torch.cuda.current_stream().synchronize()
    cc3d.sync_status()
    assert torch.equal(y8h, y8.cpu())
    p8.close()


def test_host_calls_refuse_what_they_do_not_cover():
    c, h, w = 64, 8, 8
    wt = torch.zeros((c, c, 3, 3, 3), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(c, device="cuda")
    rms = cc3d.Plan(wt, None, h=h, w=w, max_t=2, epi=cc3d.EPI_BIAS_RMS_SILU, gamma=g)
    xh = torch.zeros((1, 2, h, w, c), dtype=torch.bfloat16)
    yh = torch.zeros((1, 2, h, w, c), dtype=torch.bfloat16)
    plain = cc3d.Plan(wt, None, h=h, w=w, max_t=2)
    launches = cc3d.cc3d_launch_count()
    with pytest.raises(cc3d.Cc3dError):  # an RMS epilogue: its next caches have no host form
        rms.forward_host([dict(x_host=xh, y_host=yh)])
    with pytest.raises(cc3d.Cc3dError):  # t beyond max_t
        plain.forward_host([dict(x_host=xh, y_host=yh, t=3)])
    cache = torch.zeros((1, 2, h, w, c), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cc3d.Cc3dError):  # cache_out is cache_in
        plain.forward_host([dict(x_host=xh, y_host=yh, cache_in=cache, cache_out=cache)])
    assert cc3d.cc3d_launch_count() == launches
    rms.close()
    plain.close()

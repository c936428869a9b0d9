"""GPU parity of the downsample path's spatial step: each frame through
ZeroPad2d(0, 1, 0, 1) and a 3x3 conv with stride 2 (H x W -> H/2 x W/2),
on the tensor-core conv: the input's four stride-2 phases are loaded once
per channel chunk, each through a tensor map that walks every other pixel,
and the nine taps read them through 2 x 2 shifted views.  Cases cover 96-
and 32-channel (no-swizzle slab) and 64-channel (swizzled) chunks, one CTA
per tile, the CTA pair, two sub-tiles (the encoder's full-size layer), and
the residual epilogue."""
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu

PAD = (0, 1, 0, 1)  # ZeroPad2d(left, right, top, bottom)


def _case(n, cin, cout, t, h, w, seed):
    x = synth.normal((n, cin, t, h, w), seed)
    wt = synth.kaiming_uniform(cout, cin, (1, 3, 3), seed + 1)
    b = synth.uniform((cout,), -0.1, 0.1, seed + 2)
    return x, wt, b


def _plan(wt, b, n, h, w, t, **kw):
    return cc3d.Plan(to_dev(wt), to_dev(b), n=n, h=h, w=w, max_t=t, pad=(0, 0), stride_hw=2, **kw)


CASES = [
    # (n, c_in, c_out, t, h, w, shape): shape = (mma_ctas, tile_w, w_resident)
    (1, 96, 96, 2, 20, 24, (1, 8, 0)),
    (1, 96, 96, 2, 96, 160, (1, 8, 0)),
    (1, 64, 128, 1, 32, 48, (2, 16, 0)),
    (1, 32, 64, 2, 20, 24, (1, 8, 0)),
    (2, 192, 192, 2, 30, 52, (2, 16, 0)),
]


@pytest.mark.parametrize("n,cin,cout,t,h,w,shape", CASES)
def test_stride2_spatial_conv_matches_oracle(n, cin, cout, t, h, w, shape):
    x, wt, b = _case(n, cin, cout, t, h, w, cin + cout + h)
    plan = _plan(wt, b, n, h, w, t)
    st = plan.stats()
    assert (st.mma_ctas, st.tile_w, st.w_resident) == shape, "tile shape"
    xd = to_dev(synth.ndhwc(x))
    y = torch.empty((n, t, h // 2, w // 2, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(xd, y)
    cc3d.sync_status()
    ref = oracle.conv2d_frames(synth.ncthw_view(xd.cpu()), wt[:, :, 0], b.double().numpy(),
                               stride=(2, 2), pad=PAD)
    assert_close_bf16(ncthw_np(y), ref, f"stride-2 conv n{n} {cin}->{cout} {h}x{w}")


def test_stride2_spatial_conv_residual_epilogue():
    n, cin, cout, t, h, w = 1, 64, 128, 2, 32, 48
    x, wt, b = _case(n, cin, cout, t, h, w, 81)
    plan = _plan(wt, b, n, h, w, t, epi=cc3d.EPI_BIAS_RESIDUAL)
    xd = to_dev(synth.ndhwc(x))
    res = to_dev(synth.ndhwc(synth.normal((n, cout, t, h // 2, w // 2), 82)))
    y = torch.empty_like(res)
    plan.forward(xd, y, residual=res)
    cc3d.sync_status()
    ref = oracle.conv2d_frames(synth.ncthw_view(xd.cpu()), wt[:, :, 0], b.double().numpy(),
                               stride=(2, 2), pad=PAD) + ncthw_np(res)
    assert_close_bf16(ncthw_np(y), ref, "stride-2 conv + residual")


def test_encoder_downsample_full_size_crops():
    """The encoder's first downsample, x[1, 96, 17, 480, 832] -> 240 x 416
    (two sub-tiles per CTA): the oracle on crops of two frames, one at the
    top-left corner and one at the bottom-right (where the zero column and
    row after the frame are read)."""
    n, c, t, h, w = 1, 96, 17, 480, 832
    g = torch.Generator(device="cuda")
    g.manual_seed(83)
    xd = torch.randn((n, t, h, w, c), generator=g, device="cuda").to(torch.bfloat16)
    wt = synth.kaiming_uniform(c, c, (1, 3, 3), 84)
    b = synth.uniform((c,), -0.1, 0.1, 85)
    plan = _plan(wt, b, n, h, w, t)
    assert plan.stats().tile_w == 16
    y = torch.empty((n, t, h // 2, w // 2, c), dtype=torch.bfloat16, device="cuda")
    plan.forward(xd, y)
    cc3d.sync_status()
    k = 24  # output rows / columns per crop
    for fr, (i0, j0) in ((0, (0, 0)), (t - 1, (h // 2 - k, w // 2 - k))):
        rows = min(2 * k + 1, h - 2 * i0)  # input rows the crop's outputs read
        cols = min(2 * k + 1, w - 2 * j0)
        xc = xd[:, fr:fr + 1, 2 * i0:2 * i0 + rows, 2 * j0:2 * j0 + cols].cpu()
        ref = oracle.conv2d_frames(synth.ncthw_view(xc), wt[:, :, 0], b.double().numpy(),
                                   stride=(2, 2), pad=PAD)
        got = y[:, fr:fr + 1, i0:i0 + k, j0:j0 + k]
        assert_close_bf16(ncthw_np(got), ref, f"downsample crop frame {fr} at {i0},{j0}")

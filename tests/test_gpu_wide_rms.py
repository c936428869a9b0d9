"""GPU parity of the RMS_norm epilogues on rows wider than one MMA (up to
512 channels: the two CTAs of a cluster each hold one half of the row for
the same pixels and swap each row's partial sum of squares), of the RMS_norm
epilogue without SiLU, of the
stand-alone RMS_norm without SiLU, and of the downsample path they make
up ("Cosmos3 Wan VAE", §10.5: WanRMS_norm, then ZeroPad2d + 3x3 stride-2
Conv2d per frame, then WanRMS_norm).  References round a conv's output to
bf16 before its RMS_norm, as the block's reading does."""
import numpy as np
import pytest
import torch

import oracle
from tests import sampled
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


def _rms_ref(conv, g, beta=None, silu=True):
    return oracle.rms_norm(oracle.round_bf16_array(conv), g.double().numpy(),
                           None if beta is None else beta.double().numpy(), silu=silu)


# (n, c_in, c_out, t, h, w, epi)
WIDE = [
    (1, 384, 384, 2, 16, 20, cc3d.EPI_BIAS_RMS_SILU),
    (1, 96, 384, 2, 16, 20, cc3d.EPI_BIAS_RMS_SILU),
    (2, 32, 320, 2, 12, 16, cc3d.EPI_BIAS_RMS_SILU),
    (1, 64, 512, 2, 9, 17, cc3d.EPI_BIAS_RMS_SILU),
    (1, 384, 384, 3, 10, 14, cc3d.EPI_BIAS_RMS),
    (1, 64, 64, 2, 17, 20, cc3d.EPI_BIAS_RMS),
]


@pytest.mark.parametrize("n,cin,cout,t,h,w,epi", WIDE)
def test_rms_epilogues_match_oracle(n, cin, cout, t, h, w, epi):
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=cin + cout + epi)
    g = synth.uniform((cout,), 0.5, 1.5, 70)
    be = synth.uniform((cout,), -0.2, 0.2, 71)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t, epi=epi,
                     gamma=to_dev(g), beta=to_dev(be))
    st = plan.stats()
    # rows up to 256 channels: one CTA owns the whole row; wider: each CTA
    # of a cluster one half
    assert st.row_ctas == (2 if cout > 256 else 1)
    assert st.n_tile * st.row_ctas == cout
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    nc_in = to_dev(synth.ndhwc(synth.normal((n, cout, 2, h, w), 72)))
    nc_out = torch.empty_like(nc_in)
    plan.forward(x, y, next_cache_in=nc_in, next_cache_out=nc_out)
    cc3d.sync_status()
    assert torch.equal(nc_out.cpu(), y[:, -2:].cpu())
    conv = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    ref = _rms_ref(conv, g, be, silu=epi == cc3d.EPI_BIAS_RMS_SILU)
    assert_close_bf16(ncthw_np(y), ref, f"rms epilogue {cin}->{cout} epi{epi}")


def test_wide_rms_many_tiles_per_cluster():
    """The block's 384-channel shape, [1, 384, 5, 60, 104]: each cluster
    takes several M tiles in turn, so both exchange slots and both phases of
    their barriers are reused; checked at seeded voxels of every frame plus
    every border pixel of the last frame, against the oracle's conv at those
    voxels (all channels), rounded to bf16 and RMS-normalised."""
    n, c, t, h, w = 1, 384, 5, 60, 104
    case = synth.conv_case(c, c, t, h, w, n=n, seed_base=84)
    g = synth.uniform((c,), 0.5, 1.5, 85)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t,
                     epi=cc3d.EPI_BIAS_RMS_SILU, gamma=to_dev(g))
    assert plan.stats().row_ctas == 2
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, c), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    vox = sampled.random_voxels(t, h, w, 400, 86)
    vox[t - 1] = np.concatenate([vox.get(t - 1, np.zeros((0, 2), np.int32)),
                                 sampled.border_pixels(h, w)])
    got, ref = [], []
    for f, hw in sorted(vox.items()):
        s = max(0, f - 2)
        pts = np.concatenate([np.zeros((len(hw), 1), np.int32),
                              np.full((len(hw), 1), f - s, np.int32), hw], axis=1)
        conv = oracle.causal_conv3d_points(synth.ncthw_view(x[:1, s:f + 1].cpu()), case["w"],
                                           case["b"].double().numpy(), None, pts)
        # [P, C] -> [1, C, 1, 1, P]: the RMS_norm over channels of each voxel
        conv5 = np.ascontiguousarray(conv.T.reshape(1, c, 1, 1, -1))
        ref.append(_rms_ref(conv5, g).reshape(c, -1).T)
        ih = torch.as_tensor(hw[:, 0], dtype=torch.long, device="cuda")
        iw = torch.as_tensor(hw[:, 1], dtype=torch.long, device="cuda")
        got.append(y[0, f][ih, iw].double().cpu().numpy())
    assert_close_bf16(np.concatenate(got), np.concatenate(ref), "wide rms, block shape")


def test_wide_rms_streaming_is_bitwise_whole():
    n, c, t, h, w = 1, 384, 3, 12, 20
    case = synth.conv_case(c, c, t, h, w, n=n, seed_base=73)
    g = synth.uniform((c,), 0.5, 1.5, 74)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t,
                     epi=cc3d.EPI_BIAS_RMS_SILU, gamma=to_dev(g))
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, c), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    caches = [torch.empty((n, 2, h, w, c), dtype=torch.bfloat16, device="cuda") for _ in (0, 1)]
    ys, cache = [], None
    for s in range(t):
        yc = torch.empty((n, 1, h, w, c), dtype=torch.bfloat16, device="cuda")
        plan.forward(x[:, s:s + 1].contiguous(), yc, cache_in=cache, cache_out=caches[s % 2])
        cache = caches[s % 2]
        ys.append(yc)
    cc3d.sync_status()
    assert torch.equal(torch.cat(ys, dim=1).cpu(), y.cpu())


@pytest.mark.parametrize("c", [96, 384])
def test_standalone_rms_norm_with_cache(c):
    n, t, h, w = 1, 3, 9, 14
    x = synth.normal((n, c, t, h, w), 75)
    g = synth.uniform((c,), 0.5, 1.5, 76)
    be = synth.uniform((c,), -0.2, 0.2, 77)
    xd = to_dev(synth.ndhwc(x))
    y = torch.empty_like(xd)
    c_in = to_dev(synth.ndhwc(synth.normal((n, c, 2, h, w), 78)))
    c_out = torch.empty_like(c_in)
    cc3d.rms(xd, to_dev(g), y, beta=to_dev(be), cache_in=c_in, cache_out=c_out)
    y1 = torch.empty((n, 1, h, w, c), dtype=torch.bfloat16, device="cuda")
    c1 = torch.empty_like(c_in)
    cc3d.rms(xd[:, :1].contiguous(), to_dev(g), y1, beta=to_dev(be), cache_in=c_in, cache_out=c1)
    cc3d.sync_status()
    ref = oracle.rms_norm(synth.ncthw_view(xd.cpu()), g.double().numpy(), be.double().numpy(),
                          silu=False)
    assert_close_bf16(ncthw_np(y), ref, f"rms_norm c{c}")
    assert torch.equal(c_out.cpu(), y[:, -2:].cpu())
    assert torch.equal(c1[:, :1].cpu(), c_in[:, 1:].cpu())
    assert torch.equal(c1[:, 1:].cpu(), y1.cpu())


@pytest.mark.parametrize("c,h,w", [(96, 32, 48), (64, 30, 52)])
def test_downsample_path_matches_oracle(c, h, w):
    """WanRMS_norm -> ZeroPad2d(0, 1, 0, 1) + 3x3 stride-2 conv -> WanRMS_norm:
    the first norm stand-alone, the second in the conv's epilogue."""
    n, t = 1, 2
    x = synth.normal((n, c, t, h, w), 79)
    ga = synth.uniform((c,), 0.5, 1.5, 80)
    gb = synth.uniform((c,), 0.5, 1.5, 81)
    wt = synth.kaiming_uniform(c, c, (1, 3, 3), 82)
    b = synth.uniform((c,), -0.1, 0.1, 83)
    xd = to_dev(synth.ndhwc(x))
    a = torch.empty_like(xd)
    cc3d.rms(xd, to_dev(ga), a)
    plan = cc3d.Plan(to_dev(wt), to_dev(b), n=n, h=h, w=w, max_t=t, pad=(0, 0), stride_hw=2,
                     epi=cc3d.EPI_BIAS_RMS, gamma=to_dev(gb))
    y = torch.empty((n, t, h // 2, w // 2, c), dtype=torch.bfloat16, device="cuda")
    plan.forward(a, y)
    cc3d.sync_status()
    a_ref = oracle.round_bf16_array(oracle.rms_norm(synth.ncthw_view(xd.cpu()),
                                                    ga.double().numpy(), silu=False))
    conv = oracle.conv2d_frames(a_ref, wt[:, :, 0], b.double().numpy(), stride=(2, 2),
                                pad=(0, 1, 0, 1))
    ref = _rms_ref(conv, gb, silu=False)
    assert_close_bf16(ncthw_np(a), a_ref, "downsample: first norm")
    assert_close_bf16(ncthw_np(y), ref, "downsample path")

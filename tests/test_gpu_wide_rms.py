"""GPU parity of the RMS_norm epilogues on rows wider than one MMA (up to
512 channels: the CTA tile holds the whole row as two MMAs of half the
width per K step), of the RMS_norm epilogue without SiLU, of the
stand-alone RMS_norm without SiLU, and of the downsample path they make
up ("Cosmos3 Wan VAE", §10.5: WanRMS_norm, then ZeroPad2d + 3x3 stride-2
Conv2d per frame, then WanRMS_norm).  References round a conv's output to
bf16 before its RMS_norm, as the block's reading does."""
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


def _rms_ref(conv, g, beta=None, silu=True):
    return oracle.rms_norm(oracle.round_bf16_array(conv), g.double().numpy(),
                           None if beta is None else beta.double().numpy(), silu=silu)


# (n, c_in, c_out, t, h, w, epi, mma_ctas)
WIDE = [
    (1, 384, 384, 2, 16, 20, cc3d.EPI_BIAS_RMS_SILU, 2),
    (1, 96, 384, 2, 16, 20, cc3d.EPI_BIAS_RMS_SILU, 1),
    (2, 32, 320, 2, 12, 16, cc3d.EPI_BIAS_RMS_SILU, None),
    (1, 384, 384, 3, 10, 14, cc3d.EPI_BIAS_RMS, 2),
    (1, 64, 64, 2, 17, 20, cc3d.EPI_BIAS_RMS, None),
]


@pytest.mark.parametrize("n,cin,cout,t,h,w,epi,ctas", WIDE)
def test_rms_epilogues_match_oracle(n, cin, cout, t, h, w, epi, ctas):
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=cin + cout + epi)
    g = synth.uniform((cout,), 0.5, 1.5, 70)
    be = synth.uniform((cout,), -0.2, 0.2, 71)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t, epi=epi,
                     gamma=to_dev(g), beta=to_dev(be))
    st = plan.stats()
    assert st.n_tile == cout, "one CTA tile owns the whole row"
    if ctas is not None:
        assert st.mma_ctas == ctas
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

"""GPU parity of the causal conv kernels against the fp64 oracle, called
through the C ABI (ctypes binding).  Inputs are seeded (synth); the oracle
reads the same bf16 values through a channels-last view."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import (assert_close_bf16, assert_close_fp32, gather_points, ncthw_np,
                          to_dev)
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


def _bias64(b):
    return b.double().numpy()


def run_conv(case, t_chunk=None, cache=None, epi=cc3d.EPI_BIAS, **kw):
    x = to_dev(synth.ndhwc(case["x"]))
    n, t, h, w, _ = x.shape
    co = case["w"].shape[0]
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t, epi=epi, **kw)
    y = torch.empty((n, t, h, w, co), dtype=x.dtype, device="cuda")
    plan.forward(x, y, cache_in=cache)
    cc3d.sync_status()
    return plan, x, y


SMALL = [
    # (c_in, c_out, t, h, w)  -- several tiles and ragged tails in h and w
    (64, 64, 3, 20, 13),
    (32, 48, 2, 17, 9),
    (96, 96, 3, 33, 17),
    (128, 384, 2, 16, 24),
    (192, 192, 2, 18, 10),
    (64, 256, 1, 7, 5),
]


@pytest.mark.parametrize("cin,cout,t,h,w", SMALL)
def test_umma_conv_matches_oracle(cin, cout, t, h, w):
    case = synth.conv_case(cin, cout, t, h, w, seed_base=cin + cout)
    plan, x, y = run_conv(case)
    assert plan.stats().variant == cc3d.VARIANT_UMMA
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], _bias64(case["b"]))
    assert_close_bf16(ncthw_np(y), ref, f"conv {cin}->{cout} t{t} {h}x{w}")


def test_umma_conv_with_cache_and_cache_out():
    cin, cout, t, h, w = 64, 64, 3, 19, 11
    case = synth.conv_case(cin, cout, t, h, w, seed_base=5)
    cache = synth.normal((1, cin, 2, h, w), 77)
    cache_d = to_dev(synth.ndhwc(cache))
    x = to_dev(synth.ndhwc(case["x"]))
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), h=h, w=w, max_t=t)
    y = torch.empty((1, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    cache_out = torch.full_like(cache_d, 7.0)
    plan.forward(x, y, cache_in=cache_d, cache_out=cache_out)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], _bias64(case["b"]),
                               cache=synth.ncthw_view(cache_d.cpu()))
    assert_close_bf16(ncthw_np(y), ref, "conv with cache")
    # cache_out = last 2 frames of concat(cache_in, x), bit for bit
    assert torch.equal(cache_out.cpu(), x.cpu()[:, t - 2:t])


def test_cache_out_for_one_frame_chunk_rolls_window():
    cin, h, w = 32, 9, 8
    case = synth.conv_case(cin, 32, 1, h, w, seed_base=9)
    cache = to_dev(synth.ndhwc(synth.normal((1, cin, 2, h, w), 78)))
    x = to_dev(synth.ndhwc(case["x"]))
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), h=h, w=w, max_t=1)
    y = torch.empty((1, 1, h, w, 32), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(cache)
    plan.forward(x, y, cache_in=cache, cache_out=out)
    torch.cuda.synchronize()
    assert torch.equal(out[:, 0].cpu(), cache[:, 1].cpu())
    assert torch.equal(out[:, 1].cpu(), x[:, 0].cpu())
    # no cache: the window starts with a zero frame
    plan.forward(x, y, cache_in=None, cache_out=out)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[:, 0]).item() == 0
    assert torch.equal(out[:, 1].cpu(), x[:, 0].cpu())


def _stream_chunks(plan, x, chunk, cin):
    n, t, h, w, _ = x.shape
    co = plan.desc.c_out
    ys = []
    cache = None
    bufs = [torch.empty((n, 2, h, w, cin), dtype=x.dtype, device="cuda") for _ in range(2)]
    for k, s in enumerate(range(0, t, chunk)):
        xc = x[:, s:s + chunk].contiguous()
        yc = torch.empty((n, xc.shape[1], h, w, co), dtype=x.dtype, device="cuda")
        nxt = bufs[k % 2]
        plan.forward(xc, yc, cache_in=cache, cache_out=nxt)
        cache = nxt
        ys.append(yc)
    cc3d.sync_status()
    return torch.cat(ys, dim=1)


def test_config2_whole_and_streaming_bitwise_and_oracle():
    """Decoder latent-res conv, C 384 -> 384 on [1,384,5,30,52]: whole
    sequence vs 5 one-frame chunks with a 2-frame cache, identical bytes;
    both against the full fp64 oracle.  The plan's tiles (for 5-frame calls)
    are one CTA per tile; its second tile choice, CTA pairs with their own
    weight image, runs the one-frame calls and also this uncached
    whole-sequence call, whose cheap first frames balance the pair tiles'
    second round."""
    case = synth.conv_case(384, 384, 5, 30, 52)
    plan, x, y = run_conv(case)
    st = plan.stats()
    assert st.k_split == 1  # every output sums all taps in one accumulator
    assert (st.mma_ctas, st.one_frame_mma_ctas) == (1, 2)
    assert st.second_tile_calls == 1  # (run_conv's whole-sequence call)
    ys = _stream_chunks(plan, x, 1, 384)
    assert torch.equal(ys.cpu(), y.cpu()), "streaming != whole sequence"
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], _bias64(case["b"]))
    assert_close_bf16(ncthw_np(y), ref, "config 2")
    # a 5-frame call with a cache (zeros: the same conv) runs on the plan's
    # own tiles and gives the same bytes
    before = plan.stats().second_tile_calls
    zeros = torch.zeros((1, 2, 30, 52, 384), dtype=torch.bfloat16, device="cuda")
    y_c = torch.empty_like(y)
    plan.forward(x, y_c, cache_in=zeros)
    cc3d.sync_status()
    assert plan.stats().second_tile_calls == before
    assert torch.equal(y_c.cpu(), y.cpu()), "own tiles != second tiles"


def test_config2_streaming_plan_is_bitwise_the_whole_sequence_plan():
    """The config-2 layer planned for one-frame calls only (max_t = 1) may
    pick another tile shape than the plan for 5-frame calls; every output
    still sums its taps into one accumulator in the same order, so its
    streamed chunks give the whole-sequence plan's bytes."""
    case = synth.conv_case(384, 384, 5, 30, 52)
    plan5, x, y = run_conv(case)
    plan1 = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), h=30, w=52, max_t=1)
    assert plan1.stats().k_split == 1
    ys = _stream_chunks(plan1, x, 1, 384)
    assert torch.equal(ys.cpu(), y.cpu()), "streaming-only plan != whole-sequence plan"


@pytest.mark.parametrize("chunk", [2, 3])
def test_streaming_multi_frame_chunks_bitwise(chunk):
    case = synth.conv_case(64, 96, 7, 21, 18, seed_base=3)
    plan, x, y = run_conv(case)
    ys = _stream_chunks(plan, x, chunk, 64)
    assert torch.equal(ys.cpu(), y.cpu())


def test_determinism_two_runs_identical_bytes():
    case = synth.conv_case(128, 128, 3, 24, 16, seed_base=4)
    plan, x, y = run_conv(case)
    y2 = torch.empty_like(y)
    plan.forward(x, y2)
    cc3d.sync_status()
    assert torch.equal(y.cpu(), y2.cpu())


def test_causality_on_gpu():
    case = synth.conv_case(64, 64, 5, 16, 16, seed_base=6)
    plan, x, y = run_conv(case)
    x2 = x.clone()
    x2[:, 3] = torch.randn_like(x2[:, 3].float()).to(x2.dtype)
    y2 = torch.empty_like(y)
    plan.forward(x2, y2)
    cc3d.sync_status()
    assert torch.equal(y2[:, :3].cpu(), y[:, :3].cpu())
    assert not torch.equal(y2[:, 3].cpu(), y[:, 3].cpu())


def test_bias_once_zero_input():
    case = synth.conv_case(64, 80, 2, 10, 9, seed_base=8)
    case["x"] = torch.zeros_like(case["x"])
    plan, x, y = run_conv(case)
    exp = case["b"].to(torch.bfloat16)
    assert torch.equal(y.cpu(), exp.expand_as(y.cpu()))


def test_fp32_config1_matches_oracle():
    """fp32 causal conv: x[1,16,5,16,16] ~ N(0,1) seed 0, Kaiming W, bias
    U(-0.1, 0.1); within 1e-4 relative."""
    case = synth.conv_case(16, 16, 5, 16, 16, dtype=torch.float32)
    x = to_dev(synth.ndhwc(case["x"]))
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), h=16, w=16, max_t=5, dtype=cc3d.FP32)
    assert plan.stats().variant == cc3d.VARIANT_FP32
    y = torch.empty((1, 5, 16, 16, 16), dtype=torch.float32, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(case["x"], case["w"], _bias64(case["b"]))
    assert_close_fp32(ncthw_np(y), ref, "config 1")


def test_residual_epilogue():
    case = synth.conv_case(64, 64, 2, 17, 11, seed_base=12)
    res = synth.normal((1, 64, 2, 17, 11), 55)
    r_d = to_dev(synth.ndhwc(res))
    x = to_dev(synth.ndhwc(case["x"]))
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), h=17, w=11, max_t=2,
                     epi=cc3d.EPI_BIAS_RESIDUAL)
    y = torch.empty_like(r_d)
    plan.forward(x, y, residual=r_d)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], _bias64(case["b"]))
    ref = ref + res.double().numpy()
    assert_close_bf16(ncthw_np(y), ref, "residual epilogue")


def test_rms_silu_epilogue():
    c = 192
    case = synth.conv_case(c, c, 2, 18, 9, seed_base=13)
    g = synth.uniform((c,), 0.5, 1.5, 66)
    x = to_dev(synth.ndhwc(case["x"]))
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), h=18, w=9, max_t=2,
                     epi=cc3d.EPI_BIAS_RMS_SILU, gamma=to_dev(g))
    y = torch.empty((1, 2, 18, 9, c), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    h1 = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], _bias64(case["b"]))
    # the conv's output is rounded to bf16 before its RMS_norm (the block's h1)
    ref = oracle.rms_norm(oracle.round_bf16_array(h1), g.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "rms+silu epilogue")


def test_sampled_points_config3b_shape():
    """96 -> 96 at full resolution 17 x 480 x 832 (the encoder's first
    resblock conv), checked on sampled voxels: frames 0, 1, 2, T-1 at random
    pixels plus random voxels."""
    cin = cout = 96
    t, h, w = 17, 480, 832
    case = synth.conv_case(cin, cout, t, h, w)
    plan, x, y = run_conv(case)
    pts = synth.sample_points(1, t, h, w, 2048, 123)
    edge = synth.sample_points(1, t, h, w, 0, 0, frames=[0])[::997]
    pts = torch.cat([pts, edge])
    ref = oracle.causal_conv3d_points(synth.ncthw_view(x.cpu()), case["w"], _bias64(case["b"]),
                                      None, pts)
    got = gather_points(y.cpu(), pts)
    assert_close_bf16(got, ref, "config 3b sampled")


# ---- thin first layer (C_in <= 8) --------------------------------------------------

# (w * cin % 8 == 0: the halo by TMA, else staged with plain loads; RGB
# 3x3x3 takes the kernel-row-shifted A buffer, the others the im2col tile)
@pytest.mark.parametrize("cin,cout,t,h,w", [(3, 96, 3, 20, 13), (3, 96, 3, 35, 24),
                                            (3, 32, 2, 17, 9), (1, 16, 2, 9, 8),
                                            (8, 64, 2, 16, 11), (4, 48, 2, 18, 14)])
def test_thin_conv_matches_oracle(cin, cout, t, h, w):
    case = synth.conv_case(cin, cout, t, h, w, seed_base=30 + cin, x_dist="uniform")
    plan, x, y = run_conv(case)
    assert plan.stats().variant == cc3d.VARIANT_THIN
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], _bias64(case["b"]))
    assert_close_bf16(ncthw_np(y), ref, f"thin conv {cin}->{cout}")


def test_thin_conv_with_cache_and_streaming_bitwise():
    cin, cout, t, h, w = 3, 96, 4, 19, 10
    case = synth.conv_case(cin, cout, t, h, w, seed_base=44, x_dist="uniform")
    plan, x, y = run_conv(case)
    ys = _stream_chunks(plan, x, 1, cin)
    assert torch.equal(ys.cpu(), y.cpu())
    cache = to_dev(synth.ndhwc(synth.uniform((1, cin, 2, h, w), -1, 1, 45, torch.bfloat16)))
    y2 = torch.empty_like(y)
    plan.forward(x, y2, cache_in=cache)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], _bias64(case["b"]),
                               cache=synth.ncthw_view(cache.cpu()))
    assert_close_bf16(ncthw_np(y2), ref, "thin conv with cache")


def test_config3_encoder_chain_sampled():
    """Video x[1,3,17,480,832] ~ U(-1,1) -> causal conv 3 -> 96 -> causal conv
    96 -> 96, full size.  Each layer is checked on sampled voxels with the
    oracle fed the same inputs that layer saw (layer 2 gets the GPU's bf16
    output of layer 1)."""
    t, h, w = 17, 480, 832
    c1 = synth.conv_case(3, 96, t, h, w, x_dist="uniform")
    plan1, x, y1 = run_conv(c1)
    assert plan1.stats().variant == cc3d.VARIANT_THIN
    w2 = synth.kaiming_uniform(96, 96, (3, 3, 3), 11)
    b2 = synth.uniform((96,), -0.1, 0.1, 12)
    plan2 = cc3d.Plan(to_dev(w2), to_dev(b2), h=h, w=w, max_t=t)
    y2 = torch.empty_like(y1)
    plan2.forward(y1, y2)
    cc3d.sync_status()
    pts = torch.cat([synth.sample_points(1, t, h, w, 3000, 77),
                     synth.sample_points(1, t, h, w, 0, 0, frames=[0, t - 1])[::2011]])
    x_cpu, y1_cpu, y2_cpu = x.cpu(), y1.cpu(), y2.cpu()
    ref1 = oracle.causal_conv3d_points(synth.ncthw_view(x_cpu), c1["w"], _bias64(c1["b"]), None,
                                       pts)
    assert_close_bf16(gather_points(y1_cpu, pts), ref1, "config 3a sampled")
    ref2 = oracle.causal_conv3d_points(synth.ncthw_view(y1_cpu), w2, _bias64(b2), None, pts)
    assert_close_bf16(gather_points(y2_cpu, pts), ref2, "config 3b (chained) sampled")

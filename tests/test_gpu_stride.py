"""GPU parity of the temporal-stride-2 causal conv (the downsample path's
time_conv, stride (2, 1, 1)): output frame t reads input frames 2t, 2t+1,
2t+2 of the front-padded (or cached) sequence, so T input frames give
(T-1)//2 + 1 output frames.  The cases cover every tile shape the plan can
pick (one MMA tile, two sub-tiles, the CTA pair, resident weights), each
asserted through the plan's stats, odd and even T, a cache, the residual
and RMS epilogues, and streaming in 2-frame chunks, which must reproduce
the whole-sequence call bit for bit."""
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, gather_points, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu

S = 2

CASES = [
    # (n, c_in, c_out, t, h, w, k, shape): shape = (mma_ctas, tile_w, k_split)
    (8, 32, 48, 3, 20, 150, (3, 3, 3), (1, 8, 1)),
    (8, 32, 48, 4, 20, 150, (3, 3, 3), (1, 8, 1)),
    (4, 32, 384, 5, 17, 92, (3, 1, 1), (1, 16, 1)),
    (16, 64, 128, 5, 16, 40, (3, 1, 1), (2, 16, 1)),
    (1, 64, 64, 9, 20, 36, (3, 1, 1), (2, 16, 1)),
    (1, 32, 48, 8, 20, 30, (3, 3, 3), (1, 8, 1)),
]


def t_out(t):
    return (t - 1) // S + 1


def _plan(case, n, h, w, max_t, **kw):
    return cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=max_t,
                     stride_t=S, **kw)


def _shape(plan):
    st = plan.stats()
    return (st.mma_ctas, st.tile_w, st.k_split)


def _ref(x, case, k, cache=None):
    return oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                                cache=cache, pad=(k[1] // 2, k[2] // 2), stride_t=S)


def _stream(plan, x, chunks, n, h, w, cin, cout, residual=None):
    """Runs x as consecutive chunks of the given input-frame counts, each
    carrying the last two input frames of the one before."""
    caches = [torch.empty((n, 2, h, w, cin), dtype=torch.bfloat16, device="cuda")
              for _ in range(2)]
    cache_in, start, out_start, ys = None, 0, 0, []
    for i, c in enumerate(chunks):
        yc = torch.empty((n, t_out(c), h, w, cout), dtype=torch.bfloat16, device="cuda")
        res = None
        if residual is not None:
            res = residual[:, out_start:out_start + t_out(c)].contiguous()
        plan.forward(x[:, start:start + c].contiguous(), yc, cache_in=cache_in,
                     cache_out=caches[i % 2], residual=res)
        cache_in = caches[i % 2]
        start += c
        out_start += t_out(c)
        ys.append(yc)
    cc3d.sync_status()
    return torch.cat(ys, dim=1)


@pytest.mark.parametrize("n,cin,cout,t,h,w,k,shape", CASES)
def test_stride2_conv_matches_oracle(n, cin, cout, t, h, w, k, shape):
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=cin + 3 * cout + t)
    plan = _plan(case, n, h, w, t)
    assert _shape(plan) == shape, f"tile shape {_shape(plan)}"
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t_out(t), h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    assert_close_bf16(ncthw_np(y), _ref(x, case, k), f"stride 2 n{n} {cin}->{cout} t{t} k{k}")


@pytest.mark.parametrize("n,cin,cout,t,h,w,k,shape",
                         [CASES[0], CASES[3], CASES[5]])
def test_stride2_with_cache_matches_oracle(n, cin, cout, t, h, w, k, shape):
    """A cache of two real frames: output frame 0 reads both of them."""
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=cin + cout + 91)
    cache = synth.normal((n, cin, 2, h, w), 92)
    plan = _plan(case, n, h, w, t)
    assert _shape(plan) == shape
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t_out(t), h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y, cache_in=to_dev(synth.ndhwc(cache)))
    cc3d.sync_status()
    ref = _ref(x, case, k, cache=cache.double().numpy())
    assert_close_bf16(ncthw_np(y), ref, "stride 2 with cache")


@pytest.mark.parametrize("idx,chunks", [(2, [2, 2, 1]), (3, [2, 2, 1]), (4, [2, 2, 2, 2, 1]),
                                        (5, [2, 4, 2])])
def test_stride2_streaming_is_bitwise_whole(idx, chunks):
    """Chunks of an even frame count (the last one may be odd) give the
    whole-sequence outputs exactly, on every tile shape."""
    n, cin, cout, t, h, w, k, shape = CASES[idx]
    assert sum(chunks) == t
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=cin + cout + 17)
    plan = _plan(case, n, h, w, t)
    assert _shape(plan) == shape
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t_out(t), h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    ys = _stream(plan, x, chunks, n, h, w, cin, cout)
    assert ys.shape == y.shape
    assert torch.equal(ys.cpu(), y.cpu())


def test_stride2_residual_epilogue_and_streaming():
    n, cin, cout, t, h, w, k = 1, 64, 96, 5, 21, 18, (3, 3, 3)
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=93)
    plan = _plan(case, n, h, w, t, epi=cc3d.EPI_BIAS_RESIDUAL)
    assert _shape(plan) == (2, 16, 1)
    x = to_dev(synth.ndhwc(case["x"]))
    res = to_dev(synth.ndhwc(synth.normal((n, cout, t_out(t), h, w), 94)))
    y = torch.empty_like(res)
    plan.forward(x, y, residual=res)
    ys = _stream(plan, x, [2, 2, 1], n, h, w, cin, cout, residual=res)
    assert torch.equal(ys.cpu(), y.cpu())
    ref = _ref(x, case, k) + ncthw_np(res)
    assert_close_bf16(ncthw_np(y), ref, "stride 2 residual")


def test_stride2_rms_epilogue_and_next_cache():
    """RMS_norm + SiLU epilogue on the output frames; next_cache_out holds
    the last two of them (after the carried frames of next_cache_in)."""
    n, cin, cout, t, h, w, k = 1, 64, 128, 5, 20, 36, (3, 3, 3)
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=95)
    g = synth.uniform((cout,), 0.5, 1.5, 96)
    plan = _plan(case, n, h, w, t, epi=cc3d.EPI_BIAS_RMS_SILU, gamma=to_dev(g))
    assert _shape(plan) == (2, 16, 1)
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t_out(t), h, w, cout), dtype=torch.bfloat16, device="cuda")
    nc_in = to_dev(synth.ndhwc(synth.normal((n, cout, 2, h, w), 97)))
    nc_out = torch.empty_like(nc_in)
    plan.forward(x, y, next_cache_in=nc_in, next_cache_out=nc_out)
    # a one-output chunk: next_cache_out = (last carried frame, its output)
    y1 = torch.empty((n, 1, h, w, cout), dtype=torch.bfloat16, device="cuda")
    nc1 = torch.empty_like(nc_in)
    plan.forward(x[:, :2].contiguous(), y1, next_cache_in=nc_in, next_cache_out=nc1)
    cc3d.sync_status()
    assert torch.equal(nc_out.cpu(), y[:, -2:].cpu())
    assert torch.equal(nc1[:, :1].cpu(), nc_in[:, 1:].cpu())
    assert torch.equal(nc1[:, 1:].cpu(), y1.cpu())
    assert torch.equal(y1.cpu(), y[:, :1].cpu())
    conv = _ref(x, case, k)
    ref = oracle.rms_norm(oracle.round_bf16_array(conv), g.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "stride 2 rms epilogue")


def test_stride2_time_conv_full_size_sampled():
    """The time_conv shape of the downsample path at full size (192 channels,
    17 frames of 120 x 208, kernel (3, 1, 1)): the first and last output
    frames and seeded voxels against the oracle, and eight 2-frame chunks
    plus a final 1-frame chunk against the whole-sequence call, bit for bit."""
    n, c, t, h, w, k = 1, 192, 17, 120, 208, (3, 1, 1)
    case = synth.conv_case(c, c, t, h, w, n=n, k=k, seed_base=98)
    plan = _plan(case, n, h, w, t)
    st = plan.stats()
    assert (st.mma_ctas, st.w_resident) == (2, 1), "expected the pair with resident weights"
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t_out(t), h, w, c), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    ys = _stream(plan, x, [2] * 8 + [1], n, h, w, c, c)
    assert torch.equal(ys.cpu(), y.cpu())
    pts = synth.sample_points(n, t_out(t), h, w, 512, 99, frames=[0, t_out(t) - 1])
    got = gather_points(y.cpu(), pts)
    ref = oracle.causal_conv3d_points(synth.ncthw_view(x.cpu()), case["w"],
                                      case["b"].double().numpy(), None, pts, pad=(0, 0),
                                      stride_t=S)
    assert_close_bf16(got, ref, "time_conv full size sampled")

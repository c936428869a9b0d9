"""GPU parity of small frames (fewer tiles than SMs), where every output
still sums all of its taps in one accumulator, and of the frame caches the
conv kernel writes itself (cache_out: the last kt-1 input frames of
concat(cache_in, x); next_cache_out: the last two output frames of the RMS
epilogue), on each tile shape the planner picks for them."""
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


def _run(n, cin, cout, t, h, w, seed, cache=None, epi=cc3d.EPI_BIAS, gamma=None):
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=seed)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t, epi=epi,
                     gamma=gamma)
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y, cache_in=cache)
    cc3d.sync_status()
    return case, plan, x, y


@pytest.mark.parametrize("n", [1, 20])
def test_small_frames_match_oracle(n):
    cin, cout, t, h, w = 64, 64, 3, 17, 9
    case, plan, x, y = _run(n, cin, cout, t, h, w, seed=50 + n)
    assert plan.stats().k_split == 1
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    assert_close_bf16(ncthw_np(y), ref, f"n={n}")


def test_small_frame_with_cache_every_tap_from_a_real_frame():
    """With a cache no tap of the first frames is a causal zero frame."""
    n, cin, cout, t, h, w = 2, 96, 192, 2, 20, 30
    cache = synth.normal((n, cin, 2, h, w), 61)
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=60)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t)
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y, cache_in=to_dev(synth.ndhwc(cache)))
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                               cache=cache.double().numpy())
    assert_close_bf16(ncthw_np(y), ref, "small frame with cache")


def test_rms_epilogue_small_frame():
    c, t, h, w = 192, 3, 18, 9
    g = synth.uniform((c,), 0.5, 1.5, 62)
    case, plan, x, y = _run(1, c, c, t, h, w, seed=63, epi=cc3d.EPI_BIAS_RMS_SILU,
                            gamma=to_dev(g))
    conv = oracle.round_bf16_array(
        oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy()))
    ref = oracle.rms_norm(conv, g.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "small-frame rms epilogue")


def test_residual_epilogue_and_cuda_graph_replay():
    """Residual epilogue on a small frame, called eagerly and from a CUDA
    graph of the same calls (one-frame chunks carrying the cache): same bytes."""
    n, cin, cout, t, h, w = 1, 64, 96, 3, 21, 18
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=64)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t,
                     epi=cc3d.EPI_BIAS_RESIDUAL)
    x = to_dev(synth.ndhwc(case["x"]))
    res = to_dev(synth.ndhwc(synth.normal((n, cout, t, h, w), 65)))
    xs = [x[:, s:s + 1].contiguous() for s in range(t)]
    rs = [res[:, s:s + 1].contiguous() for s in range(t)]
    caches = [torch.empty((n, 2, h, w, cin), dtype=torch.bfloat16, device="cuda")
              for _ in range(2)]

    def run(ys):
        cache = None
        for s in range(t):
            plan.forward(xs[s], ys[s], cache_in=cache, cache_out=caches[s % 2], residual=rs[s])
            cache = caches[s % 2]

    eager = [torch.empty((n, 1, h, w, cout), dtype=torch.bfloat16, device="cuda")
             for _ in range(t)]
    run(eager)
    cc3d.sync_status()
    graphed = [torch.full_like(e, float("nan")) for e in eager]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(graphed)
    g.replay()
    torch.cuda.synchronize()
    cc3d.sync_status()
    for a, b in zip(eager, graphed):
        assert torch.equal(a.cpu(), b.cpu())
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    ref = ref + ncthw_np(res)
    assert_close_bf16(ncthw_np(torch.cat(eager, dim=1)), ref, "small-frame residual")


# (n, c_in, c_out, h, w, max_t, k): one MMA tile with two N tiles, two
# sub-tiles, a CTA pair with two N tiles, a ragged frame, a 3x1x1 kernel
CACHE_CASES = [
    (2, 384, 384, 30, 52, 5, (3, 3, 3)),
    (8, 32, 48, 20, 150, 1, (3, 3, 3)),
    (1, 128, 384, 17, 28, 1, (3, 3, 3)),
    (1, 64, 64, 17, 9, 3, (3, 3, 3)),
    (1, 64, 64, 20, 36, 5, (3, 1, 1)),
]


@pytest.mark.parametrize("n,cin,cout,h,w,max_t,k", CACHE_CASES)
def test_cache_out_written_by_the_conv(n, cin, cout, h, w, max_t, k):
    """cache_out = the last two frames of concat(cache_in or zeros, x), for
    one-frame calls with and without a cache and for a longer call, every
    byte; and the conv's own output is unaffected by writing it."""
    t = max_t
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=cin + cout + h)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=max_t)
    x = to_dev(synth.ndhwc(case["x"]))
    cache_in = to_dev(synth.ndhwc(synth.normal((n, cin, 2, h, w), 66)))
    junk = lambda: torch.full((n, 2, h, w, cin), 7.0, dtype=torch.bfloat16, device="cuda")  # noqa
    y1 = torch.empty((n, 1, h, w, cout), dtype=torch.bfloat16, device="cuda")
    c_a, c_b = junk(), junk()
    plan.forward(x[:, :1].contiguous(), y1, cache_in=cache_in, cache_out=c_a)
    plan.forward(x[:, :1].contiguous(), y1, cache_out=c_b)
    cc3d.sync_status()
    assert torch.equal(c_a[:, :1].cpu(), cache_in[:, 1:].cpu())
    assert torch.equal(c_a[:, 1:].cpu(), x[:, :1].cpu())
    assert torch.equal(c_b[:, :1].cpu(), torch.zeros_like(c_b[:, :1]).cpu())
    assert torch.equal(c_b[:, 1:].cpu(), x[:, :1].cpu())
    if t >= 2:
        y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
        y_plain = torch.empty_like(y)
        c_c = junk()
        plan.forward(x, y, cache_in=cache_in, cache_out=c_c)
        plan.forward(x, y_plain, cache_in=cache_in)
        cc3d.sync_status()
        assert torch.equal(c_c.cpu(), x[:, t - 2:].cpu())
        assert torch.equal(y.cpu(), y_plain.cpu())

"""GPU parity of the temporal split (a cluster of kt CTAs per output tile,
one temporal tap each, the partial sums added in the last CTA through
distributed shared memory) and of the unsplit path at the same small frame
sizes.  The plan splits when kt CTAs per tile still fit one wave, so the
batch size decides which path a small frame takes; each case asserts it."""
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


@pytest.mark.parametrize("n,split", [(1, 3), (20, 1)])
def test_split_and_unsplit_match_oracle(n, split):
    cin, cout, t, h, w = 64, 64, 3, 17, 9
    case, plan, x, y = _run(n, cin, cout, t, h, w, seed=50 + n)
    st = plan.stats()
    assert st.k_split == split
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    assert_close_bf16(ncthw_np(y), ref, f"n={n} split={split}")


def test_split_with_cache_every_tap_from_a_real_frame():
    """With a cache no sender's tap is a zero frame: all three partials are
    exchanged on every tile."""
    n, cin, cout, t, h, w = 2, 96, 192, 2, 20, 30
    cache = synth.normal((n, cin, 2, h, w), 61)
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=60)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t)
    assert plan.stats().k_split == 3
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y, cache_in=to_dev(synth.ndhwc(cache)))
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                               cache=cache.double().numpy())
    assert_close_bf16(ncthw_np(y), ref, "split with cache")


def test_rms_epilogue_small_frame_runs_unsplit():
    """RMS_norm + SiLU needs whole rows in one CTA: a small frame with this
    epilogue keeps one CTA per tile."""
    c, t, h, w = 192, 3, 18, 9
    g = synth.uniform((c,), 0.5, 1.5, 62)
    case, plan, x, y = _run(1, c, c, t, h, w, seed=63, epi=cc3d.EPI_BIAS_RMS_SILU,
                            gamma=to_dev(g))
    assert plan.stats().k_split == 1
    conv = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    ref = oracle.rms_norm(conv, g.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "small-frame rms epilogue")


def test_split_residual_epilogue_and_cuda_graph_replay():
    """Residual epilogue on the split path, called eagerly and from a CUDA
    graph of the same calls (one-frame chunks carrying the cache): same bytes."""
    n, cin, cout, t, h, w = 1, 64, 96, 3, 21, 18
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=64)
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t,
                     epi=cc3d.EPI_BIAS_RESIDUAL)
    assert plan.stats().k_split == 3
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
    assert_close_bf16(ncthw_np(torch.cat(eager, dim=1)), ref, "split residual")

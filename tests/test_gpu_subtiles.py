"""GPU parity of the two-sub-tile UMMA configuration (a 16 x 16 pixel CTA tile
made of two 8 x 16 MMA tiles that share every weight stage).  The plan picks
it from the tile waves of one frame (times the batch), so these cases use
batch sizes that select it at sizes the oracle finishes in seconds; each
asserts the choice through the plan's stats."""
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu

SUB2 = [
    # (n, c_in, c_out, t, h, w, k): w % 16 == 6 leaves the second sub-tile of
    # the last tile column wholly outside the frame, w % 16 == 12 partly
    (8, 32, 48, 1, 20, 150, (3, 3, 3)),
    (4, 32, 384, 1, 17, 92, (3, 3, 3)),
    (8, 64, 64, 2, 20, 150, (1, 1, 1)),
    (8, 64, 64, 3, 18, 146, (3, 1, 1)),
]


def _plan(case, n, h, w, t, **kw):
    return cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t, **kw)


@pytest.mark.parametrize("n,cin,cout,t,h,w,k", SUB2)
def test_two_subtile_conv_matches_oracle(n, cin, cout, t, h, w, k):
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=cin + cout + k[0])
    plan = _plan(case, n, h, w, t)
    assert plan.stats().tile_w == 16, "expected the two-sub-tile configuration"
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                               pad=(k[1] // 2, k[2] // 2))
    assert_close_bf16(ncthw_np(y), ref, f"sub2 conv n{n} {cin}->{cout} {h}x{w} k{k}")


def test_two_subtile_residual_and_streaming_bitwise():
    n, cin, cout, t, h, w = 8, 32, 48, 3, 20, 150
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=9)
    plan = _plan(case, n, h, w, t, epi=cc3d.EPI_BIAS_RESIDUAL)
    assert plan.stats().tile_w == 16
    x = to_dev(synth.ndhwc(case["x"]))
    res = to_dev(synth.ndhwc(synth.normal((n, cout, t, h, w), 31)))
    y = torch.empty_like(res)
    plan.forward(x, y, residual=res)
    # the same sequence as one-frame chunks carrying a 2-frame cache
    mk = lambda: torch.empty((n, 2, h, w, cin), dtype=torch.bfloat16, device="cuda")  # noqa: E731
    caches = [mk(), mk()]
    cache_in = None
    ys = []
    for s in range(t):
        yc = torch.empty((n, 1, h, w, cout), dtype=torch.bfloat16, device="cuda")
        plan.forward(x[:, s:s + 1].contiguous(), yc, cache_in=cache_in, cache_out=caches[s % 2],
                     residual=res[:, s:s + 1].contiguous())
        cache_in = caches[s % 2]
        ys.append(yc)
    cc3d.sync_status()
    assert torch.equal(torch.cat(ys, dim=1).cpu(), y.cpu())
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    ref = ref + ncthw_np(res)
    assert_close_bf16(ncthw_np(y), ref, "sub2 residual")


def test_two_subtile_rms_epilogue():
    """RMS_norm + SiLU epilogue over two sub-tiles of 128 channels each."""
    n, cin, cout, t, h, w = 37, 32, 128, 2, 17, 32
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=11)
    g = synth.uniform((cout,), 0.5, 1.5, 12)
    plan = _plan(case, n, h, w, t, epi=cc3d.EPI_BIAS_RMS_SILU, gamma=to_dev(g))
    assert plan.stats().tile_w == 16
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    conv = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy())
    ref = oracle.rms_norm(oracle.round_bf16_array(conv), g.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "sub2 rms epilogue")

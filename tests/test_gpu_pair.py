"""GPU parity of the CTA-pair path: a cluster of two CTAs on one SM pair
takes a 16 x 16 pixel tile, each CTA loading its own 8 x 16 half of the
halo and half of every weight stage, and the first CTA issues 2-SM
tcgen05 MMAs (M = 256) into both CTAs' tensor memory.  The plan picks it
for 64-channel chunks when its tile waves are cheaper; each case asserts
the choice (mma_ctas == 2) and compares every output with the oracle."""
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu

PAIR = [
    # (n, c_in, c_out, t, h, w, k): w % 16 == 9 puts one valid column in the
    # second CTA's half of the last tile column, w % 16 == 8 none (its whole
    # half lies outside the frame), w % 16 == 12 four
    (20, 64, 64, 2, 17, 9, (3, 3, 3)),
    (6, 64, 192, 2, 20, 40, (3, 3, 3)),
    (4, 128, 384, 1, 17, 28, (3, 3, 3)),
    (8, 64, 64, 2, 18, 22, (1, 1, 1)),
    (16, 64, 128, 3, 16, 40, (3, 1, 1)),
]


def _plan(case, n, h, w, t, **kw):
    return cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t, **kw)


@pytest.mark.parametrize("n,cin,cout,t,h,w,k", PAIR)
def test_pair_conv_matches_oracle(n, cin, cout, t, h, w, k):
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=cin + cout + 7 * k[0])
    plan = _plan(case, n, h, w, t)
    st = plan.stats()
    assert (st.mma_ctas, st.tile_w, st.k_split) == (2, 16, 1), "expected the CTA-pair path"
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                               pad=(k[1] // 2, k[2] // 2))
    assert_close_bf16(ncthw_np(y), ref, f"pair conv n{n} {cin}->{cout} {h}x{w} k{k}")


def test_pair_residual_cache_and_streaming_bitwise():
    n, cin, cout, t, h, w = 6, 64, 192, 3, 20, 40
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=71)
    plan = _plan(case, n, h, w, t, epi=cc3d.EPI_BIAS_RESIDUAL)
    assert plan.stats().mma_ctas == 2
    x = to_dev(synth.ndhwc(case["x"]))
    res = to_dev(synth.ndhwc(synth.normal((n, cout, t, h, w), 72)))
    y = torch.empty_like(res)
    plan.forward(x, y, residual=res)
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
    assert_close_bf16(ncthw_np(y), ref + ncthw_np(res), "pair residual")


def test_pair_rms_epilogue_with_cache():
    n, cin, cout, t, h, w = 6, 64, 128, 2, 20, 40
    case = synth.conv_case(cin, cout, t, h, w, n=n, seed_base=73)
    g = synth.uniform((cout,), 0.5, 1.5, 74)
    plan = _plan(case, n, h, w, t, epi=cc3d.EPI_BIAS_RMS_SILU, gamma=to_dev(g))
    assert plan.stats().mma_ctas == 2
    cache = synth.normal((n, cin, 2, h, w), 75)
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y, cache_in=to_dev(synth.ndhwc(cache)))
    cc3d.sync_status()
    conv = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                                cache=cache.double().numpy())
    ref = oracle.rms_norm(oracle.round_bf16_array(conv), g.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "pair rms epilogue with cache")

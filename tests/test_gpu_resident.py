"""GPU parity of the resident-weight mode: with a 1 x 1 spatial kernel
(kernel (kt, 1, 1): the downsample path's time_conv, a 1 x 1 x 1 conv) and a
single N tile, every weight stage of a CTA is loaded into a shared-memory
slot of its own once per launch and read in place by the MMAs of every
tile, instead of streaming through the weight ring once per tile.  The
cases cover one CTA per tile (32- and 96-channel chunks) and the CTA pair,
each asserted through the plan's stats, with a cache, streaming, and the
residual and RMS epilogues."""
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu

RESIDENT = [
    # (n, c_in, c_out, t, h, w, k, mma_ctas)
    (8, 32, 64, 3, 20, 150, (1, 1, 1), 1),
    (8, 32, 64, 3, 20, 150, (3, 1, 1), 1),
    (2, 96, 192, 3, 20, 70, (3, 1, 1), 1),
    (2, 96, 192, 3, 20, 70, (1, 1, 1), 1),
    (6, 64, 192, 2, 20, 40, (1, 1, 1), 2),
    (4, 64, 64, 3, 20, 36, (3, 1, 1), 2),
]


def _plan(case, n, h, w, t, **kw):
    return cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t, **kw)


@pytest.mark.parametrize("n,cin,cout,t,h,w,k,ctas", RESIDENT)
def test_resident_weights_match_oracle(n, cin, cout, t, h, w, k, ctas):
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=cin + cout + 5 * k[0])
    plan = _plan(case, n, h, w, t)
    st = plan.stats()
    assert (st.w_resident, st.mma_ctas, st.k_split) == (1, ctas, 1), "expected resident weights"
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                               pad=(0, 0))
    assert_close_bf16(ncthw_np(y), ref, f"resident n{n} {cin}->{cout} k{k}")


@pytest.mark.parametrize("idx", [1, 2, 5])
def test_resident_cache_and_streaming_bitwise(idx):
    """A cache of two real frames, then the same sequence as one-frame
    chunks: the chunks reproduce the whole call bit for bit."""
    n, cin, cout, t, h, w, k, ctas = RESIDENT[idx]
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=cin + cout + 71)
    cache = synth.normal((n, cin, 2, h, w), 72)
    plan = _plan(case, n, h, w, t)
    assert plan.stats().w_resident == 1
    x = to_dev(synth.ndhwc(case["x"]))
    c_dev = to_dev(synth.ndhwc(cache))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y, cache_in=c_dev)
    bufs = [torch.empty((n, 2, h, w, cin), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    cache_in, ys = c_dev, []
    for s in range(t):
        yc = torch.empty((n, 1, h, w, cout), dtype=torch.bfloat16, device="cuda")
        plan.forward(x[:, s:s + 1].contiguous(), yc, cache_in=cache_in, cache_out=bufs[s % 2])
        cache_in = bufs[s % 2]
        ys.append(yc)
    cc3d.sync_status()
    assert torch.equal(torch.cat(ys, dim=1).cpu(), y.cpu())
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                               cache=cache.double().numpy(), pad=(0, 0))
    assert_close_bf16(ncthw_np(y), ref, "resident with cache")


def test_resident_residual_epilogue():
    n, cin, cout, t, h, w, k, _ = RESIDENT[3]
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=73)
    plan = _plan(case, n, h, w, t, epi=cc3d.EPI_BIAS_RESIDUAL)
    assert plan.stats().w_resident == 1
    x = to_dev(synth.ndhwc(case["x"]))
    res = to_dev(synth.ndhwc(synth.normal((n, cout, t, h, w), 74)))
    y = torch.empty_like(res)
    plan.forward(x, y, residual=res)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                               pad=(0, 0)) + ncthw_np(res)
    assert_close_bf16(ncthw_np(y), ref, "resident residual")


def test_resident_rms_epilogue_on_a_pair():
    n, cin, cout, t, h, w, k, _ = RESIDENT[5]
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=75)
    g = synth.uniform((cout,), 0.5, 1.5, 76)
    be = synth.uniform((cout,), -0.2, 0.2, 77)
    plan = _plan(case, n, h, w, t, epi=cc3d.EPI_BIAS_RMS_SILU, gamma=to_dev(g), beta=to_dev(be))
    st = plan.stats()
    assert (st.w_resident, st.mma_ctas) == (1, 2)
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty((n, t, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    cc3d.sync_status()
    conv = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                                pad=(0, 0))
    ref = oracle.rms_norm(oracle.round_bf16_array(conv), g.double().numpy(),
                          be.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "resident rms epilogue")

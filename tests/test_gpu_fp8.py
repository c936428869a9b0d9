"""GPU parity of the FP8 (E4M3) causal conv ("Cosmos3 Wan VAE", §9 names
low-precision conv quantisation; E4M3 is the FP8 form the tensor cores
take): the activation quantiser bit for bit against the oracle's (both
divide in fp32 and round once to E4M3), and the conv on E4M3 operands,
y = s_x * s_w[co] * conv(q_x, q_w) + b[co], against the oracle's conv on
the same codes, on each tile shape the planner picks for FP8, with a cache,
the temporal stride 2 and the residual epilogue, and streamed chunks of
E4M3 codes bit for bit equal to the whole sequence."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


def _scales(x, w):
    """Synthetic calibration: amax / 448 per tensor (x) and per output
    channel (w), as float32 values both sides use."""
    s_x = np.float32(float(x.abs().max()) / 448.0)
    s_w = (w.float().abs().reshape(w.shape[0], -1).max(dim=1).values / 448.0).numpy()
    return float(s_x), s_w.astype(np.float32)


def _quantize_dev(x_ndhwc_dev, s_x):
    q = torch.empty(x_ndhwc_dev.shape, dtype=torch.uint8, device="cuda")
    cc3d.quantize_e4m3(x_ndhwc_dev, s_x, q)
    return q


def _codes_to_values(q_ndhwc_cpu):
    return q_ndhwc_cpu.view(torch.float8_e4m3fn).to(torch.float64)


def test_quantizer_matches_oracle_bitwise():
    g = torch.Generator().manual_seed(90)
    x = torch.cat([torch.randn(40000, generator=g) * 3, torch.rand(8000, generator=g) * 4000 - 2000,
                   torch.randn(8000, generator=g) * 1e-3]).to(torch.bfloat16)
    for s in (0.0137, 0.5, 3.7):
        q = _quantize_dev(to_dev(x), s)
        torch.cuda.synchronize()
        got = _codes_to_values(q.cpu()).numpy()
        ref = oracle.quantize_e4m3(x.float().numpy(), s, quotient="f32")
        np.testing.assert_array_equal(got, ref)


# (n, c_in, c_out, t, h, w, k, stride_t, cache, epi, mma_ctas)
CASES = [
    (1, 384, 384, 2, 30, 52, (3, 3, 3), 1, True, cc3d.EPI_BIAS, 2),
    (1, 128, 128, 2, 12, 20, (3, 3, 3), 1, False, cc3d.EPI_BIAS, 2),
    (1, 384, 384, 5, 30, 52, (3, 3, 3), 1, False, cc3d.EPI_BIAS, 1),
    (1, 128, 64, 3, 16, 20, (3, 3, 3), 2, True, cc3d.EPI_BIAS_RESIDUAL, None),
    (1, 256, 128, 5, 20, 36, (3, 1, 1), 2, False, cc3d.EPI_BIAS, None),
]


@pytest.mark.parametrize("n,cin,cout,t,h,w,k,stride,cache,epi,ctas", CASES)
def test_fp8_conv_matches_oracle(n, cin, cout, t, h, w, k, stride, cache, epi, ctas):
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=cin + cout + t)
    s_x, s_w = _scales(case["x"], case["w"])
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t, epi=epi,
                     dtype=cc3d.FP8_E4M3, w_scale=to_dev(torch.from_numpy(s_w)), x_scale=s_x,
                     stride_t=stride)
    st = plan.stats()
    assert st.variant == cc3d.VARIANT_UMMA and st.k_chunk == 128
    if ctas is not None:
        assert st.mma_ctas == ctas
    xq = _quantize_dev(to_dev(synth.ndhwc(case["x"])), s_x)
    c = synth.normal((n, cin, 2, h, w), 91) if cache else None
    cq = _quantize_dev(to_dev(synth.ndhwc(c)), s_x) if cache else None
    t_out = (t - 1) // stride + 1
    res = to_dev(synth.ndhwc(synth.normal((n, cout, t_out, h, w), 92))) \
        if epi == cc3d.EPI_BIAS_RESIDUAL else None
    y = torch.empty((n, t_out, h, w, cout), dtype=torch.bfloat16, device="cuda")
    cache_out = torch.empty((n, 2, h, w, cin), dtype=torch.uint8, device="cuda")
    plan.forward(xq, y, cache_in=cq, cache_out=cache_out, residual=res)
    cc3d.sync_status()
    # the conv's input cache: the last two frames of concat(cache_in, x), as codes
    full = torch.cat([cq.cpu(), xq.cpu()], dim=1) if cache else torch.cat(
        [torch.zeros((n, 2, h, w, cin), dtype=torch.uint8), xq.cpu()], dim=1)
    assert torch.equal(cache_out.cpu(), full[:, -2:])
    # the oracle quantises the same bf16 values itself (the quantisers agree
    # code for code: test_quantizer_matches_oracle_bitwise)
    ref = oracle.causal_conv3d_fp8(case["x"].float().numpy(), case["w"].float().numpy(),
                                   case["b"].double().numpy(), s_x, s_w,
                                   cache=c.float().numpy() if cache else None,
                                   pad=(k[1] // 2, k[2] // 2), quotient="f32", stride_t=stride)
    if res is not None:
        ref = ref + ncthw_np(res)
    assert_close_bf16(ncthw_np(y), ref, f"fp8 conv {cin}->{cout} k{k} s{stride}")


def test_fp8_streaming_is_bitwise_whole():
    n, c, t, h, w = 1, 128, 4, 14, 20
    case = synth.conv_case(c, c, t, h, w, n=n, seed_base=93)
    s_x, s_w = _scales(case["x"], case["w"])
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t,
                     dtype=cc3d.FP8_E4M3, w_scale=to_dev(torch.from_numpy(s_w)), x_scale=s_x)
    xq = _quantize_dev(to_dev(synth.ndhwc(case["x"])), s_x)
    y = torch.empty((n, t, h, w, c), dtype=torch.bfloat16, device="cuda")
    plan.forward(xq, y)
    caches = [torch.empty((n, 2, h, w, c), dtype=torch.uint8, device="cuda") for _ in (0, 1)]
    ys, cache = [], None
    for s in range(t):
        yc = torch.empty((n, 1, h, w, c), dtype=torch.bfloat16, device="cuda")
        plan.forward(xq[:, s:s + 1].contiguous(), yc, cache_in=cache, cache_out=caches[s % 2])
        cache = caches[s % 2]
        ys.append(yc)
    cc3d.sync_status()
    assert torch.equal(torch.cat(ys, dim=1).cpu(), y.cpu())


def test_fp8_plan_rejects_what_it_does_not_cover():
    w = torch.zeros((96, 96, 3, 3, 3), dtype=torch.bfloat16, device="cuda")
    s = torch.ones(96, device="cuda")
    with pytest.raises(cc3d.Cc3dError):
        cc3d.Plan(w, None, h=8, w=8, max_t=1, dtype=cc3d.FP8_E4M3, w_scale=s, x_scale=1.0)
    w = torch.zeros((128, 128, 3, 3, 3), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cc3d.Cc3dError):  # no activation scale
        cc3d.Plan(w, None, h=8, w=8, max_t=1, dtype=cc3d.FP8_E4M3, w_scale=s[:1].expand(128))

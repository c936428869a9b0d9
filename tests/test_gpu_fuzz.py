"""Seeded random cases across the tensor-core conv's whole descriptor space:
channel counts (32/64/96-channel chunks, N tiles up to 256, RMS rows up to
512), kernel shapes 3x3x3 / 3x1x1 / 1x3x3 / 1x1x1, temporal stride 1 and 2,
batch, ragged frames, every epilogue (bias, residual, RMS_norm + SiLU,
RMS_norm), a carried cache or none -- whatever tile shape the planner picks
for each -- against the fp64 oracle.  The case list is drawn once from a
fixed seed on the host (a pure function of the seed), so a failing case is
reproducible from its id."""
import random

import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu

KERNELS = [(3, 3, 3), (3, 1, 1), (1, 3, 3), (1, 1, 1)]
EPIS = [cc3d.EPI_BIAS, cc3d.EPI_BIAS_RESIDUAL, cc3d.EPI_BIAS_RMS_SILU, cc3d.EPI_BIAS_RMS]
# multiply-accumulates the oracle may spend on one case
MAC_BUDGET = 60e6


def _draw_cases(count, seed):
    rng = random.Random(seed)
    cases = []
    while len(cases) < count:
        k = rng.choice(KERNELS)
        epi = rng.choice(EPIS)
        cin = rng.choice([32, 64, 96, 128, 192])
        if epi in (cc3d.EPI_BIAS_RMS_SILU, cc3d.EPI_BIAS_RMS):
            cout = rng.choice([32, 64, 96, 128, 192, 256, 320, 384, 512])
        else:
            cout = 16 * rng.randint(1, 16)
        stride = rng.choice([1, 2]) if k[0] == 3 else 1
        n = rng.choice([1, 1, 2])
        t = rng.randint(1, 5)
        h, w = rng.randint(3, 36), rng.randint(3, 40)
        cache = k[0] > 1 and rng.random() < 0.5
        t_out = (t - 1) // stride + 1
        macs = n * t_out * h * w * cin * cout * k[0] * k[1] * k[2]
        if macs > MAC_BUDGET:
            continue
        cases.append(dict(n=n, cin=cin, cout=cout, t=t, h=h, w=w, k=k, stride=stride, epi=epi,
                          cache=cache, seed=len(cases)))
    return cases


CASES = _draw_cases(120, 20261203)


def _id(c):
    return (f"{c['seed']}-n{c['n']}-{c['cin']}to{c['cout']}-t{c['t']}-{c['h']}x{c['w']}-"
            f"k{''.join(map(str, c['k']))}-s{c['stride']}-e{c['epi']}-{'c' if c['cache'] else 'n'}")


@pytest.mark.parametrize("c", CASES, ids=[_id(c) for c in CASES])
def test_random_conv_matches_oracle(c):
    n, cin, cout, t, h, w, k = c["n"], c["cin"], c["cout"], c["t"], c["h"], c["w"], c["k"]
    epi, stride = c["epi"], c["stride"]
    base = 1000 + 17 * c["seed"]
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=base)
    rms = epi in (cc3d.EPI_BIAS_RMS_SILU, cc3d.EPI_BIAS_RMS)
    g = synth.uniform((cout,), 0.5, 1.5, base + 7) if rms else None
    be = synth.uniform((cout,), -0.2, 0.2, base + 8) if rms and c["seed"] % 2 else None
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t, epi=epi,
                     gamma=to_dev(g) if g is not None else None,
                     beta=to_dev(be) if be is not None else None, stride_t=stride)
    st = plan.stats()
    assert st.variant == cc3d.VARIANT_UMMA and st.k_split == 1
    x = to_dev(synth.ndhwc(case["x"]))
    t_out = (t - 1) // stride + 1
    front = k[0] - 1
    cache = (synth.normal((n, cin, front, h, w), base + 9) if c["cache"] else None)
    res = (synth.normal((n, cout, t_out, h, w), base + 10)
           if epi == cc3d.EPI_BIAS_RESIDUAL else None)
    y = torch.empty((n, t_out, h, w, cout), dtype=torch.bfloat16, device="cuda")
    cache_out = (torch.empty((n, front, h, w, cin), dtype=torch.bfloat16, device="cuda")
                 if front > 0 else None)
    plan.forward(x, y, cache_in=to_dev(synth.ndhwc(cache)) if cache is not None else None,
                 cache_out=cache_out, residual=to_dev(synth.ndhwc(res)) if res is not None else None)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                               cache=cache.double().numpy() if cache is not None else None,
                               pad=(k[1] // 2, k[2] // 2), stride_t=stride)
    if res is not None:
        ref = ref + res.double().numpy()
    if rms:
        ref = oracle.rms_norm(oracle.round_bf16_array(ref), g.double().numpy(),
                              be.double().numpy() if be is not None else None,
                              silu=epi == cc3d.EPI_BIAS_RMS_SILU)
    assert_close_bf16(ncthw_np(y), ref, _id(c))
    if cache_out is not None:
        # the last kt-1 frames of concat(cache_in or zeros, x)
        full = torch.cat([synth.ndhwc(cache) if cache is not None
                          else torch.zeros((n, front, h, w, cin), dtype=torch.bfloat16),
                          x.cpu()], dim=1)
        assert torch.equal(cache_out.cpu(), full[:, -front:])
    plan.close()


def _draw_fp8_cases(count, seed):
    rng = random.Random(seed)
    cases = []
    while len(cases) < count:
        k = rng.choice([(3, 3, 3), (3, 1, 1), (1, 1, 1)])
        cin, cout = rng.choice([128, 256]), 16 * rng.randint(1, 16)
        stride = rng.choice([1, 2]) if k[0] == 3 else 1
        t, h, w = rng.randint(1, 4), rng.randint(3, 30), rng.randint(3, 36)
        epi = rng.choice([cc3d.EPI_BIAS, cc3d.EPI_BIAS_RESIDUAL])
        cache = k[0] > 1 and rng.random() < 0.5
        t_out = (t - 1) // stride + 1
        if t_out * h * w * cin * cout * k[0] * k[1] * k[2] > MAC_BUDGET:
            continue
        cases.append(dict(cin=cin, cout=cout, t=t, h=h, w=w, k=k, stride=stride, epi=epi,
                          cache=cache, seed=len(cases)))
    return cases


FP8_CASES = _draw_fp8_cases(24, 20261204)


@pytest.mark.parametrize("c", FP8_CASES, ids=[_id(dict(c, n=1)) for c in FP8_CASES])
def test_random_fp8_conv_matches_oracle(c):
    """The same on E4M3 operands: x and the cache quantised by the library,
    weights at plan time; the oracle quantises the same bf16 values itself
    (the two quantisers agree code for code) and convolves the codes."""
    cin, cout, t, h, w, k, stride, epi = (c[key] for key in
                                          ("cin", "cout", "t", "h", "w", "k", "stride", "epi"))
    base = 5000 + 17 * c["seed"]
    case = synth.conv_case(cin, cout, t, h, w, k=k, seed_base=base)
    s_x = float(case["x"].float().abs().max()) / 448.0
    s_w = (case["w"].float().abs().reshape(cout, -1).max(dim=1).values / 448.0).contiguous()
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), h=h, w=w, max_t=t, epi=epi,
                     dtype=cc3d.FP8_E4M3, w_scale=to_dev(s_w), x_scale=s_x, stride_t=stride)
    xq = torch.empty((1, t, h, w, cin), dtype=torch.uint8, device="cuda")
    cc3d.quantize_e4m3(to_dev(synth.ndhwc(case["x"])), s_x, xq)
    front = k[0] - 1
    cache = synth.normal((1, cin, front, h, w), base + 9) if c["cache"] else None
    cq = None
    if cache is not None:
        cq = torch.empty((1, front, h, w, cin), dtype=torch.uint8, device="cuda")
        cc3d.quantize_e4m3(to_dev(synth.ndhwc(cache)), s_x, cq)
    t_out = (t - 1) // stride + 1
    res = (synth.normal((1, cout, t_out, h, w), base + 10)
           if epi == cc3d.EPI_BIAS_RESIDUAL else None)
    y = torch.empty((1, t_out, h, w, cout), dtype=torch.bfloat16, device="cuda")
    plan.forward(xq, y, cache_in=cq, residual=to_dev(synth.ndhwc(res)) if res is not None else None)
    cc3d.sync_status()
    ref = oracle.causal_conv3d_fp8(case["x"].float().numpy(), case["w"].float().numpy(),
                                   case["b"].double().numpy(), s_x, s_w.numpy(),
                                   cache=cache.float().numpy() if cache is not None else None,
                                   pad=(k[1] // 2, k[2] // 2), quotient="f32", stride_t=stride)
    if res is not None:
        ref = ref + res.double().numpy()
    assert_close_bf16(ncthw_np(y), ref, "fp8 " + _id(dict(c, n=1)))
    plan.close()


def test_case_list_is_a_function_of_the_seed():
    assert _draw_cases(120, 20261203) == CASES
    kinds = {(c["k"], c["epi"]) for c in CASES}
    assert len(kinds) >= 10  # the draw covers most kernel x epilogue pairs

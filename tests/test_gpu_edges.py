"""Edge cases of the conv entry point on the GPU against the fp64 oracle:
batch > 1, kernels 1x1x1 / 1x3x3 / 2x3x3, wide output channels (N tile 256,
two N tiles of 256), frames smaller than one tile, fp32 with a cache, and
the thin path with a batch."""
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, assert_close_fp32, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


def _run(cin, cout, t, h, w, *, n=1, k=(3, 3, 3), seed=0, with_cache=False, dtype=torch.bfloat16,
         x_dist="normal"):
    case = synth.conv_case(cin, cout, t, h, w, n=n, k=k, seed_base=seed, dtype=dtype,
                           x_dist=x_dist)
    x = to_dev(synth.ndhwc(case["x"]))
    front = k[0] - 1
    cache = None
    if with_cache and front > 0:
        cache = to_dev(synth.ndhwc(synth.normal((n, cin, front, h, w), seed + 50, dtype)))
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), n=n, h=h, w=w, max_t=t + 2,
                     dtype=cc3d.FP32 if dtype == torch.float32 else cc3d.BF16)
    y = torch.empty((n, t, h, w, cout), dtype=dtype, device="cuda")
    cache_out = torch.empty_like(cache) if cache is not None else None
    plan.forward(x, y, cache_in=cache, cache_out=cache_out)
    cc3d.sync_status()
    ref = oracle.causal_conv3d(synth.ncthw_view(x.cpu()), case["w"], case["b"].double().numpy(),
                               cache=synth.ncthw_view(cache.cpu()) if cache is not None else None,
                               pad=(k[1] // 2, k[2] // 2))
    if cache_out is not None:
        tail = torch.cat([cache.cpu(), x.cpu()], dim=1)[:, -front:]
        assert torch.equal(cache_out.cpu(), tail)
    return plan, y, ref


@pytest.mark.parametrize("n", [2, 3])
def test_batch_with_cache(n):
    _, y, ref = _run(64, 96, 3, 18, 11, n=n, seed=1, with_cache=True)
    assert_close_bf16(ncthw_np(y), ref, f"batch {n}")


@pytest.mark.parametrize("k", [(1, 1, 1), (1, 3, 3), (2, 3, 3), (3, 1, 1)])
def test_kernel_shapes(k):
    _, y, ref = _run(64, 128, 3, 17, 10, k=k, seed=2, with_cache=True)
    assert_close_bf16(ncthw_np(y), ref, f"kernel {k}")


@pytest.mark.parametrize("cin,cout", [(256, 256), (128, 512), (96, 160)])
def test_wide_and_odd_channel_tiles(cin, cout):
    plan, y, ref = _run(cin, cout, 2, 16, 9, seed=3)
    assert_close_bf16(ncthw_np(y), ref, f"{cin}->{cout}")
    st = plan.stats()
    assert cout % st.n_tile == 0 and st.n_tile <= 256


def test_frame_smaller_than_a_tile():
    _, y, ref = _run(32, 32, 4, 3, 5, seed=4, with_cache=True)
    assert_close_bf16(ncthw_np(y), ref, "tiny frame")


def test_fp32_with_cache():
    _, y, ref = _run(16, 16, 3, 9, 7, seed=5, with_cache=True, dtype=torch.float32)
    assert_close_fp32(ncthw_np(y), ref, "fp32 with cache")


def test_thin_batch_with_cache():
    _, y, ref = _run(3, 96, 2, 21, 16, n=2, seed=6, with_cache=True, x_dist="uniform")
    assert_close_bf16(ncthw_np(y), ref, "thin batch 2")


def test_t_below_max_t_and_rejections():
    case = synth.conv_case(32, 32, 2, 8, 8, seed_base=7)
    x = to_dev(synth.ndhwc(case["x"]))
    plan = cc3d.Plan(to_dev(case["w"]), to_dev(case["b"]), h=8, w=8, max_t=4)
    y = torch.empty((1, 2, 8, 8, 32), dtype=torch.bfloat16, device="cuda")
    plan.forward(x, y)
    big = to_dev(synth.ndhwc(synth.normal((1, 32, 5, 8, 8), 8)))
    y5 = torch.empty((1, 5, 8, 8, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cc3d.Cc3dError) as e:
        plan.forward(big, y5)                  # t = 5 > max_t = 4
    assert e.value.status == cc3d.ERR_INVALID_ARG
    with pytest.raises(cc3d.Cc3dError) as e:
        plan.forward(x, x)                     # y overlapping x
    assert e.value.status == cc3d.ERR_ALIAS
    with pytest.raises(cc3d.Cc3dError) as e:
        cache = torch.empty((1, 2, 8, 8, 32), dtype=torch.bfloat16, device="cuda")
        plan.forward(x, y, cache_in=cache, cache_out=cache)   # cache_out == cache_in
    assert e.value.status == cc3d.ERR_ALIAS
    st = plan.stats()
    assert st.calls == 1 and st.rejected == 3

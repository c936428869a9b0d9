"""GPU parity of rmsnorm_silu and the residual block (C ABI) against the
fp64 oracle; streaming of the block with per-conv 2-frame caches."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, gather_points, ncthw_np, to_dev
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("c", [8, 40, 96, 192, 200, 384, 1024])
def test_rmsnorm_silu_matches_oracle(c):
    x = synth.normal((1, c, 3, 7, 9), 21)
    g = synth.uniform((c,), 0.5, 1.5, 22)
    xd = to_dev(synth.ndhwc(x))
    y = torch.empty_like(xd)
    cc3d.rms_silu(xd, to_dev(g), y)
    torch.cuda.synchronize()
    ref = oracle.rms_norm(x, g.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, f"rmsnorm_silu c={c}")


def test_rmsnorm_silu_beta_and_cache_out():
    c, h, w = 64, 5, 6
    x = synth.normal((1, c, 1, h, w), 23)
    g = synth.uniform((c,), 0.5, 1.5, 24)
    beta = synth.uniform((c,), -0.2, 0.2, 25)
    xd = to_dev(synth.ndhwc(x))
    y = torch.empty_like(xd)
    cin = to_dev(synth.ndhwc(synth.normal((1, c, 2, h, w), 26)))
    cout = torch.empty_like(cin)
    cc3d.rms_silu(xd, to_dev(g), y, beta=to_dev(beta), cache_in=cin, cache_out=cout)
    torch.cuda.synchronize()
    ref = oracle.rms_norm(x, g.double().numpy(), beta.double().numpy(), silu=True)
    assert_close_bf16(ncthw_np(y), ref, "rmsnorm_silu beta")
    assert torch.equal(cout[:, 0].cpu(), cin[:, 1].cpu())
    assert torch.equal(cout[:, 1].cpu(), y[:, 0].cpu())


def _block(case, h, w, t):
    dev = {k: to_dev(v) for k, v in case.items() if k != "x"}
    return cc3d.Block(dev["w1"], dev["b1"], dev["g1"], dev["w2"], dev["b2"], dev["g2"], h=h, w=w,
                      max_t=t)


def _np(t):
    return t.double().numpy()


@pytest.mark.parametrize("c,t,h,w", [(64, 3, 20, 12), (192, 3, 17, 10), (32, 2, 9, 9)])
def test_resblock_matches_oracle(c, t, h, w):
    case = synth.block_case(c, t, h, w, seed_base=c)
    blk = _block(case, h, w, t)
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty_like(x)
    blk.forward(x, y)
    cc3d.sync_status()
    ref = oracle.resblock(synth.ncthw_view(x.cpu()), case["w1"], _np(case["b1"]), _np(case["g1"]),
                          case["w2"], _np(case["b2"]), _np(case["g2"]))
    assert_close_bf16(ncthw_np(y), ref, f"resblock c={c}")


def test_resblock_streaming_equals_whole_bitwise():
    c, t, h, w = 64, 5, 16, 12
    case = synth.block_case(c, t, h, w, seed_base=2)
    blk = _block(case, h, w, t)
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty_like(x)
    blk.forward(x, y)
    mk = lambda: torch.empty((1, 2, h, w, c), dtype=torch.bfloat16, device="cuda")  # noqa: E731
    c1 = [mk(), mk()]
    c2 = [mk(), mk()]
    ys = []
    c1_in = c2_in = None
    for s in range(t):
        yc = torch.empty((1, 1, h, w, c), dtype=torch.bfloat16, device="cuda")
        blk.forward(x[:, s:s + 1].contiguous(), yc, cache1_in=c1_in, cache2_in=c2_in,
                    cache1_out=c1[s % 2], cache2_out=c2[s % 2])
        c1_in, c2_in = c1[s % 2], c2[s % 2]
        ys.append(yc)
    cc3d.sync_status()
    assert torch.equal(torch.cat(ys, dim=1).cpu(), y.cpu())


def test_resblock_config4_sampled():
    """Residual block at full size: x[1,192,9,240,416], checked on sampled
    voxels (frames 0 and T-1 at random pixels, plus random voxels)."""
    c, t, h, w = 192, 9, 240, 416
    case = synth.block_case(c, t, h, w)
    blk = _block(case, h, w, t)
    x = to_dev(synth.ndhwc(case["x"]))
    y = torch.empty_like(x)
    blk.forward(x, y)
    cc3d.sync_status()
    g = torch.Generator().manual_seed(3)
    pts = synth.sample_points(1, t, h, w, 160, 321)
    corner = torch.tensor([[0, 0, 0, 0], [0, t - 1, h - 1, w - 1], [0, 4, 0, w - 1],
                           [0, 8, h - 1, 0]], dtype=torch.int32)
    pts = torch.cat([pts, corner])
    del g
    ref = oracle.resblock_points(synth.ncthw_view(x.cpu()), case["w1"], _np(case["b1"]),
                                 _np(case["g1"]), case["w2"], _np(case["b2"]), _np(case["g2"]), pts)
    got = gather_points(y.cpu(), pts)
    assert_close_bf16(got, ref, "config 4 sampled")

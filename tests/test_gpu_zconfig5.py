"""Config 5 (the channel / resolution sweep) against the oracle, in the
launch configuration the benchmark times: C in {96, 192, 384} x (T, H, W)
in {(21, 90, 160), (21, 180, 320), (21, 360, 640)}, 3x3x3, the sequence run
as 21 one-frame chunks that carry a 2-frame cache through a plan made for
one-frame calls.  Full-size outputs are checked against the fp64 oracle at
8192 seeded voxels spread over all 21 frames, and in frames 0, 1, 2 and 20
at every pixel where that costs the oracle at most ~150 GFLOP (the rows
C = 96 at 90 x 160 and 180 x 320, C = 192 at 90 x 160), else at every
border pixel of those frames (where the zero padding enters) plus 256
seeded pixels each (tests/sampled.py).  Every voxel of those four frames
at C = 384 and 360 x 640 would be 7.3 TFLOP of fp64 work."""
import pytest
import torch

from tests.parity import to_dev
import numpy as np

from tests.sampled import (all_pixels, border_pixels, check_voxels, random_voxels,
                           sample_frame_points)
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu

T = 21


@pytest.mark.parametrize("h,w", [(90, 160), (180, 320), (360, 640)])
@pytest.mark.parametrize("c", [96, 192, 384])
def test_config5_streamed_chunks_match_oracle(c, h, w):
    g = torch.Generator(device="cuda")
    g.manual_seed(c * 1000 + h)
    x = torch.randn((1, T, h, w, c), generator=g, device="cuda").to(torch.bfloat16)
    wt = synth.kaiming_uniform(c, c, (3, 3, 3), 100 + c)
    b = synth.uniform((c,), -0.1, 0.1, 200 + c)
    plan = cc3d.Plan(to_dev(wt), to_dev(b), h=h, w=w, max_t=1)
    y = torch.empty_like(x)
    bufs = [torch.empty((1, 2, h, w, c), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    cache = None
    for k in range(T):
        plan.forward(x[:, k:k + 1], y[:, k:k + 1], t=1, cache_in=cache, cache_out=bufs[k % 2])
        cache = bufs[k % 2]
    cc3d.sync_status()
    frames = [0, 1, 2, T - 1]
    full = len(frames) * h * w * c * c * 27 * 2 <= 150e9
    pts = random_voxels(T, h, w, 8192, c + h)
    for k, f in enumerate(frames):
        hw = all_pixels(h, w) if full else np.concatenate(
            [border_pixels(h, w), sample_frame_points(h, w, 256, c + h + k)])
        pts[f] = np.unique(np.concatenate([pts.get(f, np.zeros((0, 2), np.int32)), hw]), axis=0)
    check_voxels(x, y, wt, b, pts, f"config 5 C={c} {h}x{w}")
